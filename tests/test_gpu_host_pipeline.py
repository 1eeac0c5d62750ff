"""Decode steps fed from host memory (``jssa_decode_host`` through ``HostPipeline``): with each
step's uploads and download overlapping the neighbouring steps' kernels, they give exactly the
outputs of the same steps run one by one on device tensors (the same kernels on the same inputs),
those outputs agree with the oracle's decode step, and the host-side checks reject bad buffers.
"""

import math

import numpy as np
import pytest
import torch

from oracle import jssa as O
from parity import Case, check_output, f64
from synth import sample_decode_queries

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from token_level_sparse_fp8_b200 import build
    build.build()


def test_host_pipeline_matches_device_steps():
    import token_level_sparse_fp8_b200 as J
    # two long contexts (sampled threshold, several scan chunks) and a ragged one
    case = Case([20000, 17001, 3000], seed=1301, calib=2048)
    budget = 512
    layer = J.PagedLayer(case.gpu(case.k_cache), case.gpu(case.v_cache), case.gpu(case.block_table),
                         case.gpu(case.seq_lens_t), case.gpu_np(case.m32), budget)
    layer.prefill_scores()
    # the new token of every step is the row already cached at position L - 1 (rewriting it
    # leaves the caches as they were, so every step sees the same caches)
    lens = np.asarray(case.seq_lens)
    bt = case.block_table.numpy()
    rows = [(bt[b, (L - 1) // case.ps], (L - 1) % case.ps) for b, L in enumerate(lens)]
    k_new = torch.stack([case.k_cache[p, s] for p, s in rows]).contiguous()
    v_new = torch.stack([case.v_cache[p, s] for p, s in rows]).contiguous()
    n_steps = 5
    qs = [sample_decode_queries(case.factors, len(lens), case.h_q // case.h_kv, case.seed, step=i)
          for i in range(n_steps)]
    q_host = [q.pin_memory() for q in qs]
    kn_host, vn_host = k_new.pin_memory(), v_new.pin_memory()
    out_host = [torch.empty(qs[0].shape, dtype=torch.bfloat16).pin_memory() for _ in range(n_steps)]

    pipe = J.HostPipeline(layer, qs[0].shape, k_new.shape)
    for i in range(n_steps):
        pipe.step(q_host[i], kn_host, vn_host, out_host[i])
    pipe.synchronize()

    kn_dev, vn_dev = k_new.cuda(), v_new.cuda()
    scale = 1.0 / math.sqrt(case.d)
    for i in range(n_steps):
        out, _, _ = layer.step(qs[i].cuda(), kn_dev, vn_dev)
        assert torch.equal(out.cpu(), out_host[i]), f"step {i}"
    # and the oracle's decode step for the last query set
    ref = O.decode_step(f64(qs[-1]), f64(k_new), f64(v_new), case.np_k, case.np_v, case.codes,
                        case.np_bt, lens, case.m32.astype(np.float64), budget, scale)
    check_output(f64(out_host[-1]), ref["out"])


def test_host_pipeline_rejects_device_and_misshaped_buffers():
    import token_level_sparse_fp8_b200 as J
    case = Case([2048], seed=1302)
    layer = J.PagedLayer(case.gpu(case.k_cache), case.gpu(case.v_cache), case.gpu(case.block_table),
                         case.gpu(case.seq_lens_t), case.gpu_np(case.m32), 128)
    layer.prefill_scores()
    q = case.q
    kv = torch.zeros((1, case.h_kv, case.d), dtype=torch.bfloat16)
    pipe = J.HostPipeline(layer, q.shape, kv.shape)
    out = torch.empty(q.shape, dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        pipe.step(q.cuda(), kv, kv, out)
    with pytest.raises(ValueError):
        pipe.step(q[:, :4].contiguous(), kv, kv, out)
    with pytest.raises(ValueError):
        pipe.step(q, kv, None, out)
    pipe.step(q, None, None, out)  # no new token
    pipe.synchronize()
    ref, _, _ = layer.step(q.cuda())
    assert torch.equal(ref.cpu(), out)
