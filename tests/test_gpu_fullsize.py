"""Parity at the full sizes and in the launch configuration that the throughput bench times.

* GQA: the 128K-context Llama-3-8B-shaped layer (32 query / 8 KV heads, d 128, 131072-token
  contexts in permuted 16-token pages, r 32, B 2048) at batch 16, one whole decode step through
  ``jssa_decode`` with a new token. Every (sequence, KV head) pair is checked for the properties
  that hold at any size (count, ascending unique in-range positions, -1 padding, the new token's
  K/V rows written in place); sampled pairs, two per KV head, are checked element by element
  against the oracle: every scoring code of the pair, the index set (tie tolerance), the
  attention output of the pair's query heads, and the dense baseline's output over every
  position. At this size a pair's scan spans 16 chunks of
  8192 positions, 128 candidate regions: the edge of the select kernel's register tier. The same
  step at batch 1 (8 pairs, all of them sampled) takes 4096-position chunks, 256 candidate
  regions per pair: the flattened register tier. The global layer of the hybrid stack (16 query
  / 8 KV heads, d 256, r 64, 64K context, batch 8, B 2048) runs through the same checks.
* MLA: the 128-head latent layer (576-dim latent rows, 64-token pages, scoring in 64 latent +
  64 rotary dimensions, B 2048) at 128K context and batch 16: the store of every scoring row,
  score + top-B, and the absorbed latent attention; two sampled sequences against the oracle,
  properties on all; and the same latent attention over every position (the layer's dense
  baseline), eight heads of the two sequences against the oracle.

Inputs come from the seeded generator (built on the GPU, copied to the host for the oracle);
the basis is the oracle's calibration. Criteria are in ``parity.py``.
"""

import math

import numpy as np
import pytest
import torch

from oracle import jssa as O
from parity import check_codes, check_output, check_selection, f64
from synth import WORKLOADS, build_paged_kv, layer_factors, sample_calibration, sample_decode_queries

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from token_level_sparse_fp8_b200 import build
    build.build()


def _check_index_properties(gi, gc, lens, budget):
    for b in range(gi.shape[0]):
        want = min(budget, int(lens[b]))
        for h in range(gi.shape[1]):
            assert gc[b, h] == want
            sel = gi[b, h, :want]
            assert np.all(gi[b, h, want:] == -1)
            assert np.all(np.diff(sel) > 0)
            if want:
                assert sel[0] >= 0 and sel[-1] < lens[b]


def _pair_rows(cache, bt_row, h, L):
    """Host copy (bf16) of rows 0..L-1 of KV head h of one sequence, [L, d]."""
    pages = bt_row[: -(-L // cache.shape[1])].long()
    return cache[pages][:, :, h].reshape(-1, cache.shape[-1])[:L].cpu()


@pytest.mark.parametrize("name,batch", [("llama128k", 16), ("llama128k", 1), ("hybrid", 8)])
def test_gqa_decode_step_full_size(name, batch):
    import token_level_sparse_fp8_b200 as J
    w = WORKLOADS[name].replace(batch=batch)  # the bench's workloads at their full sizes
    dev = torch.device("cuda")
    L, B, G, d, r, ps = w.seq_len, w.budget, w.group, w.d, w.rank, w.page_size
    f = layer_factors(w.seed, 0, w.h_kv, w.d)
    qc, kc = sample_calibration(f, 8192, G, w.seed)
    m32 = O.calibrate(f64(qc), f64(kc), r)["M"].astype(np.float32)
    kv = build_paged_kv(f, [L] * w.batch, ps, w.seed, device=dev)
    basis = torch.from_numpy(m32).to(dev)
    layer = J.PagedLayer(kv["k_cache"], kv["v_cache"], kv["block_table"], kv["seq_lens"], basis, B)
    layer.prefill_scores()
    q = sample_decode_queries(f, w.batch, G, w.seed, step=3, device=dev)
    gen = torch.Generator(device="cpu").manual_seed(77)
    k_new = torch.randn((w.batch, w.h_kv, d), generator=gen).to(torch.bfloat16)
    v_new = torch.randn((w.batch, w.h_kv, d), generator=gen).to(torch.bfloat16)
    # the oracle's inputs: the generator's rows of the sampled pairs, copied before the CUDA path
    # runs, with the new token placed at position L - 1 on the host
    bt = kv["block_table"].long()
    rng = np.random.default_rng(5)
    if w.batch >= 2:
        sampled = [(int(b), h) for h in range(w.h_kv)
                   for b in rng.choice(w.batch, size=2, replace=False)]
    else:
        sampled = [(0, h) for h in range(w.h_kv)]
    host = {}
    for b, h in sampled:
        k_rows, v_rows = _pair_rows(kv["k_cache"], bt[b], h, L), _pair_rows(kv["v_cache"], bt[b], h, L)
        k_rows[L - 1], v_rows[L - 1] = k_new[b, h], v_new[b, h]
        host[(b, h)] = (k_rows, v_rows)  # bf16 until used
    out, idx, count = layer.step(q, k_new.to(dev), v_new.to(dev))
    # the dense baseline over the same caches (the new token included), as the bench times it
    dense = layer.dense(q)
    torch.cuda.synchronize()
    assert J.device_error() == 0

    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    lens = np.full(w.batch, L)
    _check_index_properties(gi, gc, lens, B)
    # the new token's rows are in the cache at position L - 1 of every sequence
    page = bt[:, (L - 1) // ps]
    assert torch.equal(layer.k_cache[page, (L - 1) % ps].cpu(), k_new)
    assert torch.equal(layer.v_cache[page, (L - 1) % ps].cpu(), v_new)

    qn = f64(q)
    out_np = f64(out)
    dense_np = f64(dense)
    scale = 1.0 / math.sqrt(d)
    for b, h in sampled:
        k_rows, v_rows = (f64(t) for t in host.pop((b, h)))
        # the oracle's store of every position of the pair (the new token's code included),
        # against the GPU's scoring cache
        y = k_rows @ m32[h].astype(np.float64).T
        codes = O.store_codes(k_rows, m32[h])
        sc_pages = layer.score_cache[bt[b][: L // ps]][:, h].reshape(L, r).cpu().numpy()
        check_codes(sc_pages, y)
        # selection
        qbar = O.group_mean_query(qn[b], w.h_kv)[h]
        s = O.scores(codes, O.projected_query(qbar, m32[h].astype(np.float64)))
        ref = O.select_top_b(s, B)
        check_selection(gi[b, h], gc[b, h], ref, ref.shape[0], s, B)
        # attention of the pair's query heads over the oracle's own index set, and the dense
        # baseline over every position
        for g in range(G):
            i = h * G + g
            o = O.attend(qn[b, i], k_rows[ref], v_rows[ref], scale)
            check_output(out_np[b, i][None], o[None])
            o_all = O.attend(qn[b, i], k_rows, v_rows, scale)
            check_output(dense_np[b, i][None], o_all[None])


def test_mla_decode_step_full_size():
    import token_level_sparse_fp8_b200 as J
    dev = torch.device("cuda")
    batch, h_q, D, L, ps, B, r_lat = 16, 128, 576, 131072, 64, 2048, 64
    seed = 1004
    f = layer_factors(seed, 0, 1, D)
    # the basis only has to be some calibrated basis of this generator: 32 query heads suffice
    qc, kc = sample_calibration(f, 2048, 32, seed)
    cal = O.calibrate(f64(qc)[..., :512], f64(kc)[..., :512], r_lat)
    m_lat = cal["M"].astype(np.float32)                                  # [1, 64, 512]
    m_big = O.mla_scoring_basis(m_lat[0]).astype(np.float32)[None]       # the oracle's [1, 128, 576]
    del qc, kc
    kv = build_paged_kv(f, [L] * batch, ps, seed, device=dev)
    latent = kv["k_cache"].view(kv["k_cache"].shape[0], ps, D)
    del kv["v_cache"]
    bt = kv["block_table"]
    btl = bt.long()
    checked = (0, batch - 1)
    host = {b: f64(latent[btl[b]].reshape(-1, D).cpu()) for b in checked}  # before the path runs
    num_pages = latent.shape[0]
    basis = torch.from_numpy(m_lat).to(dev)
    sc = torch.zeros((num_pages, 1, ps, 128), dtype=torch.uint8, device=dev)
    flat = latent.view(num_pages * ps, 1, D)
    for p0 in range(0, num_pages, 4096):
        p1 = min(num_pages, p0 + 4096)
        slots = torch.arange(p0 * ps, p1 * ps, dtype=torch.int64, device=dev)
        J.store(flat[p0 * ps:p1 * ps], slots, basis, sc)
    q = sample_decode_queries(f, batch, h_q, seed, step=2, device=dev)
    idx, count = J.score_topk(q, basis, sc, bt, kv["seq_lens"], B)
    scale = 1.0 / math.sqrt(D)
    out = J.mla_attend(q, latent, bt, idx, count, scale)
    # the dense baseline of the latent layer: the same kernel over every position
    idx_full = torch.arange(L, dtype=torch.int32, device=dev).repeat(batch, 1).view(batch, 1, L)
    count_full = torch.full((batch, 1), L, dtype=torch.int32, device=dev)
    out_full = J.mla_attend(q, latent, bt, idx_full, count_full, scale)
    torch.cuda.synchronize()
    assert J.device_error() == 0
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    _check_index_properties(gi, gc, np.full(batch, L), B)
    qn, out_np = f64(q), f64(out)
    for b in checked:
        rows = host.pop(b)                                            # [L, 576]
        y = rows @ m_big[0].astype(np.float64).T
        codes = O.store_codes(rows, m_big[0])
        check_codes(sc[btl[b]][:, 0].reshape(L, 128).cpu().numpy(), y)
        # the latent score sums the heads; the mean ranks identically (one latent KV head)
        qbar = O.group_mean_query(qn[b], 1)[0]
        s = O.scores(codes, O.projected_query(qbar, m_big[0].astype(np.float64)))
        ref = O.select_top_b(s, B)
        check_selection(gi[b, 0], gc[b, 0], ref, ref.shape[0], s, B)
        ref_out = np.stack([O.attend(qn[b, i], rows[ref], rows[ref][:, :512], scale)
                            for i in range(h_q)])
        check_output(out_np[b], ref_out)
        # dense over all 131072 rows, for eight of the heads (each one a pass over 600 MB)
        heads = (0, 1, 31, 63, 64, 95, 126, 127)
        ref_full = np.stack([O.attend(qn[b, i], rows, rows[:, :512], scale) for i in heads])
        check_output(f64(out_full[b])[list(heads)], ref_full)
