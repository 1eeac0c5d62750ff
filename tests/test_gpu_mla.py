"""Parity of the multi-head latent attention path with the CPU oracle, through the C ABI:
the latent calibration (second moments of the head-mean latent queries and of the latent rows,
then the latent basis), the latent scoring store (576-dim rows: the library takes the latent basis
[1, 64, 512] and passes the 64 rotary dimensions through; the oracle builds the block basis
[M_lat 0; 0 I] of 128 rows), score + top-B with one latent head (d 576, r 64, 64-token pages; one
context past the sampling point, one ragged) and the absorbed latent attention over the selected
rows (32 query heads padded into one 128-head tensor-core tile; 128 and 144 heads).
Criteria are in ``parity.py``.
"""

import math

import numpy as np
import pytest
import torch

from oracle import jssa as O
from parity import check_codes, check_output, check_selection, f64
from synth import build_paged_kv, layer_factors, sample_calibration, sample_decode_queries

pytestmark = pytest.mark.gpu

H_Q, D, R_LAT, PS = 32, 576, 64, 64


@pytest.fixture(scope="module", autouse=True)
def _built():
    from token_level_sparse_fp8_b200 import build
    build.build()


def jssa():
    import token_level_sparse_fp8_b200 as J
    return J


class MlaCase:
    def __init__(self, seq_lens, seed=1500, h_q=H_Q):
        f = layer_factors(seed, 0, 1, D)
        qc, kc = sample_calibration(f, 2048, h_q, seed)
        cal = O.calibrate(f64(qc)[..., :512], f64(kc)[..., :512], R_LAT)
        self.m_lat = cal["M"].astype(np.float32)                                  # [1, 64, 512]
        # the oracle's block basis of the same float32 values
        self.m_big = O.mla_scoring_basis(self.m_lat[0]).astype(np.float32)[None]  # [1, 128, 576]
        kv = build_paged_kv(f, list(seq_lens), PS, seed, extra_pages=2)
        self.kv = kv["k_cache"]                      # [pages, 64, 1, 576]
        self.bt = kv["block_table"]
        self.lens_t = kv["seq_lens"]
        self.lens = np.asarray(seq_lens)
        self.q = sample_decode_queries(f, len(seq_lens), h_q, seed)  # [batch, h_q, 576]
        self.np_kv = f64(self.kv)
        self.np_bt = self.bt.numpy()
        num_pages = self.np_kv.shape[0]
        y = self.np_kv.reshape(-1, D) @ self.m_big[0].astype(np.float64).T
        self.ys = y.reshape(num_pages, 1, PS, 128)
        from oracle.fp8 import e4m3_encode
        self.codes = e4m3_encode(self.ys)


@pytest.fixture(scope="module")
def case():
    return MlaCase([20000, 1500])


def test_mla_store_codes(case):
    J = jssa()
    num_pages = case.kv.shape[0]
    sc = torch.zeros((num_pages, 1, PS, 128), dtype=torch.uint8, device="cuda")
    flat = case.kv.cuda().view(num_pages * PS, 1, D)
    slots = torch.arange(num_pages * PS, dtype=torch.int64, device="cuda")
    J.store(flat, slots, torch.from_numpy(case.m_lat).cuda(), sc)
    assert check_codes(sc.cpu().numpy(), case.ys) <= 8


@pytest.mark.parametrize("budget", [2048, 700])
def test_mla_score_topk(case, budget):
    J = jssa()
    idx, count = J.score_topk(case.q.cuda(), torch.from_numpy(case.m_lat).cuda(),
                              torch.from_numpy(case.codes).cuda(), case.bt.cuda(), case.lens_t.cuda(),
                              budget)
    ref_idx, ref_count, s = O.select_step(f64(case.q), case.m_big.astype(np.float64), case.codes,
                                          case.np_bt, case.lens, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(case.lens)):
        check_selection(gi[b, 0], gc[b, 0], ref_idx[b, 0], ref_count[b, 0], s[(b, 0)], budget)


@pytest.mark.parametrize("budget", [2048, 300])
def test_mla_attend(case, budget):
    J = jssa()
    ref_idx, ref_count, _ = O.select_step(f64(case.q), case.m_big.astype(np.float64), case.codes,
                                          case.np_bt, case.lens, budget)
    scale = 1.0 / math.sqrt(D)
    kv = case.kv.cuda().view(case.kv.shape[0], PS, D)
    out = J.mla_attend(case.q.cuda(), kv, case.bt.cuda(), torch.from_numpy(ref_idx).cuda(),
                       torch.from_numpy(ref_count).cuda(), scale)
    ref = O.indexed_attend_step(f64(case.q), case.np_kv, case.np_kv[..., :512], case.np_bt, ref_idx,
                                ref_count, scale)
    check_output(f64(out), ref)


@pytest.mark.parametrize("h_q", [128, 144])
def test_mla_attend_head_counts(case, h_q):
    # 128 heads fill one M = 128 tensor-core tile; 144 heads take two head blocks, the second
    # padded with zero queries (16 real heads); both split the index set several ways
    J = jssa()
    f = layer_factors(1500, 0, 1, D)
    q = sample_decode_queries(f, len(case.lens), h_q, 1501)
    budget = 2048
    ref_idx, ref_count, _ = O.select_step(f64(q), case.m_big.astype(np.float64), case.codes,
                                          case.np_bt, case.lens, budget)
    scale = 1.0 / math.sqrt(D)
    kv = case.kv.cuda().view(case.kv.shape[0], PS, D)
    out = J.mla_attend(q.cuda(), kv, case.bt.cuda(), torch.from_numpy(ref_idx).cuda(),
                       torch.from_numpy(ref_count).cuda(), scale)
    ref = O.indexed_attend_step(f64(q), case.np_kv, case.np_kv[..., :512], case.np_bt, ref_idx,
                                ref_count, scale)
    check_output(f64(out), ref)


def test_mla_short_empty_and_exact_budget():
    # an empty sequence (zeros out), one below the budget (every position), one exactly at it
    J = jssa()
    c = MlaCase([0, 100, 512], seed=1510)
    budget = 512
    idx, count = J.score_topk(c.q.cuda(), torch.from_numpy(c.m_lat).cuda(),
                              torch.from_numpy(c.codes).cuda(), c.bt.cuda(), c.lens_t.cuda(), budget)
    assert count.cpu().numpy().ravel().tolist() == [0, 100, 512]
    gi = idx.cpu().numpy()
    assert np.all(gi[0, 0] == -1)
    assert np.array_equal(gi[1, 0, :100], np.arange(100)) and np.all(gi[1, 0, 100:] == -1)
    assert np.array_equal(gi[2, 0], np.arange(512))
    scale = 1.0 / math.sqrt(D)
    kv = c.kv.cuda().view(c.kv.shape[0], PS, D)
    out = J.mla_attend(c.q.cuda(), kv, c.bt.cuda(), idx, count, scale)
    ref = O.indexed_attend_step(f64(c.q), c.np_kv, c.np_kv[..., :512], c.np_bt, gi,
                                count.cpu().numpy(), scale)
    check_output(f64(out), ref)
    assert torch.count_nonzero(out[0]).item() == 0


@pytest.mark.parametrize("h_q", [128, 32])
def test_mla_calibration(h_q):
    # the latent second moments through the library (128 heads: the mean-plane form of the Gram
    # kernel; 32 heads: also the mean-plane form, G d = 16384) and the latent basis solved at d 512
    J = jssa()
    f = layer_factors(1520, 0, 1, D)
    # (generated on the device: 128 heads of 576 dimensions are slow to mix on the host)
    qc, kc = sample_calibration(f, 700, h_q, 1520, device="cuda")
    res = O.calibrate(f64(qc)[..., :512], f64(kc)[..., :512], R_LAT)
    acc = J.Calibration(1, 512)
    acc.add_latent(qc, kc[:, 0])
    m, lam = acc.basis(R_LAT)
    torch.cuda.synchronize()
    for g, rg in ((f64(acc.gram_q), res["gram_q"]), (f64(acc.gram_k), res["gram_k"])):
        assert np.max(np.abs(g - rg)) <= 1e-5 * np.max(np.abs(rg))
    m, lam = f64(m)[0], f64(lam)[0]
    assert np.max(np.abs(m @ m.T - np.eye(R_LAT))) <= 1e-6
    a_q, a_k = O.unit_trace(res["gram_q"][0]), O.unit_trace(res["gram_k"][0])
    # the subspace of the float32 rows, as an exact projector (rounding the rows to float32 moves
    # L_marg by up to ~1e-7 either way at d 512, which says nothing about the subspace)
    basis64, _ = np.linalg.qr(m.T)
    p_gpu, p_ref = basis64 @ basis64.T, O.projector(res["M"][0])
    opt = O.l_marg(p_ref, a_q, a_k)
    assert -1e-12 <= O.l_marg(p_gpu, a_q, a_k) - opt <= 1e-7
    assert np.max(np.abs(lam - res["eigvals"][0])) <= 1e-5 * lam[0]


def test_mla_wait_timeout_then_recovery(case):
    # a wait limit of one clock cycle makes the first wait on the tensor cores run out on a correct
    # launch: the call raises the timeout flag, waits (with the default limit) for what it issued
    # and frees its tensor memory; with the default restored, the next call is correct and clean
    J = jssa()
    budget = 2048
    ref_idx, ref_count, _ = O.select_step(f64(case.q), case.m_big.astype(np.float64), case.codes,
                                          case.np_bt, case.lens, budget)
    scale = 1.0 / math.sqrt(D)
    kv = case.kv.cuda().view(case.kv.shape[0], PS, D)
    args = (case.q.cuda(), kv, case.bt.cuda(), torch.from_numpy(ref_idx).cuda(),
            torch.from_numpy(ref_count).cuda(), scale)
    J.device_error(clear=True)
    prev = J.set_wait_limit(1)
    try:
        J.mla_attend(*args)
        torch.cuda.synchronize()
    finally:
        J.set_wait_limit(0)
    assert prev == 2000000000
    assert J.device_error(clear=True) & 32  # JSSA_DEVERR_TIMEOUT
    out = J.mla_attend(*args)
    ref = O.indexed_attend_step(f64(case.q), case.np_kv, case.np_kv[..., :512], case.np_bt, ref_idx,
                                ref_count, scale)
    check_output(f64(out), ref)
    assert J.device_error(clear=True) == 0


@pytest.mark.parametrize("budget", [2048, 512])
def test_mla_decode_step(budget):
    # one whole latent decode step through jssa_mla_decode: the new latent row and its scoring code
    # are stored by the first kernel, then score + top-B and the latent attention (contexts past
    # the sampling point, ragged, below the budget, empty)
    check_decode_step(MlaCase([20000, 3001, 300, 0], seed=1530), budget)


@pytest.mark.parametrize("batch", [20, 40, 80])
def test_mla_decode_step_larger_batches(batch):
    # larger latent batches (up to more sequences than SMs for the prep and the select): 128 query
    # heads, one context past the sampling point, the rest ragged, below the budget and empty
    rng = np.random.default_rng(batch)
    lens = [17000, 0, 700] + [int(x) for x in rng.integers(1100, 2600, batch - 3)]
    check_decode_step(MlaCase(lens, seed=1540 + batch, h_q=128), 1024)


def check_decode_step(c, budget):
    J = jssa()
    lens = c.lens
    rng = np.random.default_rng(11)
    kv_new = torch.from_numpy(rng.standard_normal((len(lens), D))).to(torch.bfloat16)
    # the oracle's copies: the new row at position L - 1, its code from the oracle's store
    np_kv = c.np_kv.copy()
    codes = c.codes.copy()
    for b, L in enumerate(lens):
        if L == 0:
            continue
        page, slot = c.np_bt[b, (L - 1) // PS], (L - 1) % PS
        np_kv[page, slot, 0] = f64(kv_new[b])
        codes[page, 0, slot] = O.store_codes(f64(kv_new[b])[None], c.m_big[0])[0]
    kv = c.kv.cuda().view(c.kv.shape[0], PS, D).clone()
    sc = torch.from_numpy(c.codes).cuda().clone()
    scale = 1.0 / math.sqrt(D)
    out, idx, count = J.mla_decode(c.q.cuda(), kv_new.cuda(), kv, sc,
                                   torch.from_numpy(c.m_lat).cuda(), c.bt.cuda(), c.lens_t.cuda(),
                                   budget, scale)
    torch.cuda.synchronize()
    assert J.device_error() == 0
    assert np.array_equal(f64(kv).reshape(np_kv.shape), np_kv)
    y = np.zeros((len(lens), 128))
    gsc = sc.cpu().numpy()
    for b, L in enumerate(lens):
        if L == 0:
            continue
        page, slot = c.np_bt[b, (L - 1) // PS], (L - 1) % PS
        check_codes(gsc[page, 0, slot][None], (f64(kv_new[b]) @ c.m_big[0].astype(np.float64).T)[None])
    ref_idx, ref_count, s = O.select_step(f64(c.q), c.m_big.astype(np.float64), codes, c.np_bt,
                                          lens, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(lens)):
        check_selection(gi[b, 0], gc[b, 0], ref_idx[b, 0], ref_count[b, 0], s[(b, 0)], budget)
    ref = O.indexed_attend_step(f64(c.q), np_kv, np_kv[..., :512], c.np_bt, ref_idx, ref_count, scale)
    check_output(f64(out), ref)
    # a second step reuses the workspace: the selection clears the attention's split counters;
    # on the same caches (the new row already stored) it is bit-identical to the first
    out2, idx2, _ = J.mla_decode(c.q.cuda(), None, kv, sc, torch.from_numpy(c.m_lat).cuda(),
                                 c.bt.cuda(), c.lens_t.cuda(), budget, scale)
    check_output(f64(out2), ref)
    assert torch.equal(idx2, idx) and torch.equal(out2, out)
