"""Parity of the d = 256 / r = 64 / G = 2 instances (the global layer and the sliding-window
layers of a hybrid local/global stack: 16 query and 8 KV heads of head dim 256) with the CPU
oracle, through the C ABI. Sizes span several scan CTAs, the sampled candidate threshold
(contexts past 16384 tokens), ragged tails and a short sequence; the dense kernel runs over the
last 1024 positions (the local layers' window) and over the full context.
Criteria are in ``parity.py``.
"""

import math

import numpy as np
import pytest
import torch

from oracle import jssa as O
from parity import Case, check_codes, check_output, check_selection, f64

pytestmark = pytest.mark.gpu

HYBRID = dict(h_q=16, h_kv=8, d=256, r=64)


@pytest.fixture(scope="module", autouse=True)
def _built():
    from token_level_sparse_fp8_b200 import build
    build.build()


def jssa():
    import token_level_sparse_fp8_b200 as J
    return J


@pytest.fixture(scope="module")
def hybrid():
    # one context past the sampling point, one ragged, one below the budget
    return Case([20000, 3333, 200], seed=1300, calib=2048, extra_pages=3, **HYBRID)


def _select_oracle(case, budget):
    return O.select_step(case.np_q, case.m32.astype(np.float64), case.codes, case.np_bt,
                         case.np_lens, budget)


def test_hybrid_store_codes():
    case = Case([2048, 300], seed=1310, calib=1024, **HYBRID)
    J = jssa()
    num_pages, ps, h_kv, d = case.k_cache.shape
    sc = torch.zeros((num_pages, h_kv, ps, case.r), dtype=torch.uint8, device="cuda")
    flat = case.gpu(case.k_cache).view(num_pages * ps, h_kv, d)
    slots = torch.arange(num_pages * ps, dtype=torch.int64, device="cuda")
    J.store(flat, slots, case.gpu_np(case.m32), sc)
    assert check_codes(sc.cpu().numpy(), case.ys) <= 4


@pytest.mark.parametrize("budget", [2048, 513])
def test_hybrid_score_topk(hybrid, budget):
    J = jssa()
    idx, count = J.score_topk(hybrid.gpu(hybrid.q), hybrid.gpu_np(hybrid.m32),
                              hybrid.gpu_np(hybrid.codes), hybrid.gpu(hybrid.block_table),
                              hybrid.gpu(hybrid.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(hybrid, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(hybrid.seq_lens)):
        for h in range(hybrid.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)


def test_hybrid_indexed_attend(hybrid):
    J = jssa()
    budget = 2048
    ref_idx, ref_count, _ = _select_oracle(hybrid, budget)
    scale = 1.0 / math.sqrt(hybrid.d)
    out = J.indexed_attend(hybrid.gpu(hybrid.q), hybrid.gpu(hybrid.k_cache),
                           hybrid.gpu(hybrid.v_cache), hybrid.gpu(hybrid.block_table),
                           hybrid.gpu_np(ref_idx), hybrid.gpu_np(ref_count), scale)
    ref = O.indexed_attend_step(hybrid.np_q, hybrid.np_k, hybrid.np_v, hybrid.np_bt, ref_idx,
                                ref_count, scale)
    check_output(f64(out), ref)


@pytest.mark.parametrize("window", [1024, -1])
def test_hybrid_dense_window(hybrid, window):
    J = jssa()
    scale = 1.0 / math.sqrt(hybrid.d)
    out = J.dense_decode(hybrid.gpu(hybrid.q), hybrid.gpu(hybrid.k_cache),
                         hybrid.gpu(hybrid.v_cache), hybrid.gpu(hybrid.block_table),
                         hybrid.gpu(hybrid.seq_lens_t), scale, window)
    ref = O.dense_step(hybrid.np_q, hybrid.np_k, hybrid.np_v, hybrid.np_bt, hybrid.np_lens, scale,
                       window)
    check_output(f64(out), ref)


def test_hybrid_decode_step(hybrid):
    J = jssa()
    case = hybrid
    budget = 2048
    lens = np.asarray(case.seq_lens)
    rng = np.random.default_rng(7)
    k_new = torch.from_numpy(rng.standard_normal((len(lens), case.h_kv, case.d))).to(torch.bfloat16)
    v_new = torch.from_numpy(rng.standard_normal((len(lens), case.h_kv, case.d))).to(torch.bfloat16)
    k_cache, v_cache = case.gpu(case.k_cache).clone(), case.gpu(case.v_cache).clone()
    sc = case.gpu_np(case.codes).clone()
    scale = 1.0 / math.sqrt(case.d)
    out, idx, count = J.decode(case.gpu(case.q), k_new.cuda(), v_new.cuda(), k_cache, v_cache, sc,
                               case.gpu_np(case.m32), case.gpu(case.block_table),
                               case.gpu(case.seq_lens_t), budget, scale)
    ref = O.decode_step(case.np_q, f64(k_new), f64(v_new), case.np_k, case.np_v, case.codes,
                        case.np_bt, lens, case.m32.astype(np.float64), budget, scale)
    assert np.array_equal(f64(k_cache), ref["k_cache"])
    assert np.array_equal(f64(v_cache), ref["v_cache"])
    assert check_codes(sc.cpu().numpy(), _projections(case, ref)) <= 2
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref["count"])
    for b in range(len(lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref["idx"][b, h], ref["count"][b, h],
                            ref["scores"][(b, h)], budget)
    check_output(f64(out), ref["out"])


def _projections(case, ref):
    """float64 projections of every slot of the updated cache (for the code check)."""
    k = ref["k_cache"]
    num_pages, ps, h_kv, d = k.shape
    ys = np.zeros((num_pages, h_kv, ps, case.r))
    for h in range(h_kv):
        ys[:, h] = (k[:, :, h].reshape(-1, d) @ case.m32[h].astype(np.float64).T).reshape(
            num_pages, ps, case.r)
    return ys


def test_hybrid_calibration():
    from synth import layer_factors, sample_calibration
    J = jssa()
    h_q, h_kv, d, r = HYBRID["h_q"], HYBRID["h_kv"], HYBRID["d"], HYBRID["r"]
    f = layer_factors(1320, 0, h_kv, d)
    q, k = sample_calibration(f, 3000, h_q // h_kv, 1320)
    res = O.calibrate(f64(q), f64(k), r)
    got = J.calibrate(q.cuda(), k.cuda(), r, batch=1024)
    gq, gk = f64(got["gram_q"]), f64(got["gram_k"])
    for g, rg in ((gq, res["gram_q"]), (gk, res["gram_k"])):
        assert np.max(np.abs(g - rg)) <= 1e-5 * np.max(np.abs(rg))
    m = f64(got["M"])
    lam = f64(got["eigvals"])
    for h in range(h_kv):
        assert np.max(np.abs(m[h] @ m[h].T - np.eye(r))) <= 1e-6
        p_gpu, p_ref = O.projector(m[h]), O.projector(res["M"][h])
        assert np.max(np.abs(p_gpu - p_ref)) <= 1e-4
        a_q, a_k = O.unit_trace(res["gram_q"][h]), O.unit_trace(res["gram_k"][h])
        opt = O.l_marg(p_ref, a_q, a_k)
        # the GPU projector is built from float32 rows, so it is a projector only to about 1e-7
        # and its objective may fall on either side of the float64 optimum by a few 1e-9
        assert abs(O.l_marg(p_gpu, a_q, a_k) - opt) <= 1e-7
        assert np.max(np.abs(lam[h] - res["eigvals"][h])) <= 1e-5 * lam[h, 0]


def test_hybrid_small_pages_score_topk():
    # 8-token pages: tiles span two pages (the per-token page path of the scan and the sample)
    case = Case([18000, 999], page_size=8, seed=1330, calib=1024, extra_pages=4, **HYBRID)
    J = jssa()
    budget = 600
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(case.codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(case, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(case.seq_lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)
