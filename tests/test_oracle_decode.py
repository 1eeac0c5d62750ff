"""Pins of the oracle's decode step (store, score, select, attend, dense).

* selection against brute-force sorting in plain Python, with planted ties (ties go to the lower
  position) and ``L <= B``;
* ``r = d`` without FP8: projected scores equal the exact group-mean logits computed through
  torch's grouped-query convention (``repeat_interleave`` of KV heads), so the selection is the
  exact top-B of the mean attention logits (JSSA summary, eqs. (1)-(2) with ``P = I``);
* ``r = d`` and ``B = L``: the JSSA step reproduces dense attention exactly;
* dense attention against torch's CPU ``scaled_dot_product_attention`` (fp64, ``enable_gqa``) on
  unpaged tensors;
* page-permutation invariance: the same logical data under two page tables gives identical
  index sets and outputs;
* store with a coordinate-selecting basis equals torch's FP8 cast of the chosen coordinates;
* the scoring cache occupies r bytes per token and KV head, 6.25% of bf16 K+V at r=32, d=128
  (the figure the pages print; fixture in ``tests/golden``).
"""

import json
import os

import numpy as np
import pytest
import torch

from oracle import jssa as O
from oracle.fp8 import e4m3_encode
from synth import WORKLOADS, build_paged_kv, layer_factors, sample_calibration, sample_decode_queries
from synth.generator import logical_rows

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _np(t):
    return t.to(torch.float64).numpy() if t.dtype in (torch.bfloat16, torch.float32, torch.float16) else t.numpy()


def _small_case(seq_lens=(300, 77), h_q=8, h_kv=2, d=32, ps=16, seed=5, extra_pages=3):
    f = layer_factors(seed, 0, h_kv, d, n_shared=8)
    kv = build_paged_kv(f, list(seq_lens), ps, seed, extra_pages=extra_pages)
    q = sample_decode_queries(f, len(seq_lens), h_q // h_kv, seed)
    return f, kv, q


def _store_all(kv, m, r):
    """Scoring cache for every stored position, written with the oracle's store step."""
    k_cache = _np(kv["k_cache"])
    num_pages, ps, h_kv, d = k_cache.shape
    sc = np.zeros((num_pages, h_kv, ps, r), dtype=np.uint8)
    for h in range(h_kv):
        codes = O.store_codes(k_cache[:, :, h].reshape(-1, d), m[h])
        sc[:, h] = codes.reshape(num_pages, ps, r)
    return sc


def test_selection_bruteforce_with_ties():
    rng = np.random.default_rng(3)
    for L in (1, 2, 5, 17, 64, 200):
        for budget in (1, 3, 16, 64, 300):
            s = rng.integers(-4, 5, size=L).astype(np.float64) * 0.5  # many ties
            got = O.select_top_b(s, budget)
            ranked = sorted(range(L), key=lambda t: (-s[t], t))
            want = sorted(ranked[: min(budget, L)])
            assert got.tolist() == want


def test_r_equals_d_recovers_exact_group_mean_logits():
    f, kv, q = _small_case()
    h_kv, d = 2, 32
    g = q.shape[1] // h_kv
    rng = np.random.default_rng(9)
    bt = kv["block_table"].numpy()
    k_cache = _np(kv["k_cache"])
    qn = _np(q)
    for b, L in enumerate(kv["seq_lens"].tolist()):
        pos = np.arange(L)
        keys = logical_rows(kv["k_cache"], bt, b, pos, kv["page_size"]).to(torch.float64)  # [L, h_kv, d]
        # exact per-head logits through torch's GQA convention, then the mean over each group
        k_rep = keys.permute(1, 0, 2).repeat_interleave(g, dim=0)                           # [H_q, L, d]
        logits = torch.einsum("hd,hld->hl", q[b].to(torch.float64), k_rep)
        mean_logits = logits.view(h_kv, g, L).mean(dim=1).numpy()
        qbar = O.group_mean_query(qn[b], h_kv)
        for h in range(h_kv):
            m, _ = np.linalg.qr(rng.standard_normal((d, d)))
            m = m.T  # r = d orthonormal basis
            k_h = O.paged_rows(k_cache, bt, b, h, pos)
            s_hat = (k_h @ m.T) @ O.projected_query(qbar[h], m)   # scores without FP8
            assert np.max(np.abs(s_hat - mean_logits[h])) <= 1e-10 * np.max(np.abs(mean_logits[h]))
            for budget in (1, 10, L // 3, L):
                ref = np.sort(np.lexsort((np.arange(L), -mean_logits[h]))[: min(budget, L)])
                assert np.array_equal(O.select_top_b(s_hat, budget), ref)


def test_full_budget_reproduces_dense():
    f, kv, q = _small_case()
    h_kv, d = 2, 32
    qc, kc = sample_calibration(f, 512, q.shape[1] // h_kv, 5)
    m = O.calibrate(_np(qc), _np(kc), d)["M"]
    sc = _store_all(kv, m, d)
    lens = kv["seq_lens"].numpy()
    scale = 1 / np.sqrt(d)
    res = O.decode_step(_np(q), None, None, _np(kv["k_cache"]), _np(kv["v_cache"]), sc,
                        kv["block_table"].numpy(), lens, m, int(lens.max()), scale)
    dense = O.dense_step(_np(q), _np(kv["k_cache"]), _np(kv["v_cache"]),
                         kv["block_table"].numpy(), lens, scale)
    assert np.array_equal(res["count"], np.repeat(lens[:, None], h_kv, 1))
    assert np.max(np.abs(res["out"] - dense)) <= 1e-14


@pytest.mark.parametrize("window", [-1, 50])
def test_dense_matches_torch_sdpa(window):
    f, kv, q = _small_case()
    h_kv = 2
    bt = kv["block_table"].numpy()
    lens = kv["seq_lens"].numpy()
    scale = 0.17
    ours = O.dense_step(_np(q), _np(kv["k_cache"]), _np(kv["v_cache"]), bt, lens, scale, window)
    for b, L in enumerate(lens):
        lo = 0 if window < 0 else max(0, L - window)
        pos = np.arange(lo, L)
        k = logical_rows(kv["k_cache"], bt, b, pos, kv["page_size"]).to(torch.float64).permute(1, 0, 2)
        v = logical_rows(kv["v_cache"], bt, b, pos, kv["page_size"]).to(torch.float64).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(
            q[b].to(torch.float64)[:, None, :], k, v, scale=scale, enable_gqa=True)[:, 0]
        assert np.max(np.abs(ours[b] - ref.numpy())) <= 1e-13


def test_page_permutation_invariance():
    f = layer_factors(21, 0, 2, 32, n_shared=8)
    lens = [333, 160]
    kv1 = build_paged_kv(f, lens, 16, 21)
    q = sample_decode_queries(f, 2, 4, 21)
    # same logical rows, different physical placement: a second page table with a reversed order
    bt1 = kv1["block_table"].numpy()
    num_pages = kv1["num_pages"]
    remap = np.arange(num_pages)[::-1]
    bt2 = remap[bt1].astype(np.int32)
    inv = np.argsort(remap)
    k2 = _np(kv1["k_cache"])[inv]
    v2 = _np(kv1["v_cache"])[inv]
    qc, kc = sample_calibration(f, 512, 4, 21)
    m = O.calibrate(_np(qc), _np(kc), 8)["M"]
    sc1 = _store_all(kv1, m, 8)
    sc2 = sc1[inv]
    args = dict(budget=40, scale=0.2)
    r1 = O.decode_step(_np(q), None, None, _np(kv1["k_cache"]), _np(kv1["v_cache"]), sc1, bt1,
                       np.array(lens), m, **args)
    r2 = O.decode_step(_np(q), None, None, k2, v2, sc2, bt2, np.array(lens), m, **args)
    assert np.array_equal(r1["idx"], r2["idx"])
    assert np.array_equal(r1["out"], r2["out"])


def test_store_with_coordinate_basis_equals_torch_cast():
    f, kv, q = _small_case()
    d, r = 32, 8
    perm = np.random.default_rng(4).permutation(d)[:r]
    m = np.eye(d)[perm]
    k = kv["k_cache"][:, :, 0].reshape(-1, d)
    codes = O.store_codes(_np(k), m)
    ref = k[:, perm].to(torch.float32).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, ref)


def test_decode_step_stores_new_token():
    f, kv, q = _small_case(seq_lens=(40, 19))
    h_kv, d, r = 2, 32, 8
    qc, kc = sample_calibration(f, 256, 4, 5)
    m = O.calibrate(_np(qc), _np(kc), r)["M"]
    sc = _store_all(kv, m, r)
    k_new = np.random.default_rng(1).standard_normal((2, h_kv, d))
    v_new = np.random.default_rng(2).standard_normal((2, h_kv, d))
    bt = kv["block_table"].numpy()
    lens = kv["seq_lens"].numpy()
    res = O.decode_step(_np(q), k_new, v_new, _np(kv["k_cache"]), _np(kv["v_cache"]), sc, bt,
                        lens, m, 8, 0.2)
    for b in range(2):
        t = lens[b] - 1
        page, slot = bt[b, t // 16], t % 16
        assert np.array_equal(res["k_cache"][page, slot], k_new[b])
        for h in range(h_kv):
            assert np.array_equal(res["score_cache"][page, h, slot], e4m3_encode(m[h] @ k_new[b, h]))


def test_golden_scoring_cache_size():
    with open(os.path.join(GOLDEN, "scoring_cache_size.json")) as fh:
        g = json.load(fh)
    r, d = g["rank"], g["head_dim"]
    k = np.random.default_rng(0).standard_normal((10, d))
    codes = O.store_codes(k, np.eye(d)[:r])
    bf16_kv_bytes = k.shape[0] * 2 * d * 2  # K and V rows in bf16
    assert codes.dtype == np.uint8 and codes.nbytes / bf16_kv_bytes == g["ratio"]
    # the byte model charges r bytes per token and KV head to the scoring scan
    base = O.algorithmic_bytes(1, 1, d, 4096, 16, r, 0)
    assert base - 4 * (4096 // 16) == 4096 * r


def test_golden_config_defaults():
    with open(os.path.join(GOLDEN, "config_defaults.json")) as fh:
        g = json.load(fh)
    for d, r in g["rank_for_head_dim"].items():
        assert int(d) // 4 == r
    w = WORKLOADS["llama128k"]
    assert w.budget == g["budget"] and w.rank == w.d // 4
