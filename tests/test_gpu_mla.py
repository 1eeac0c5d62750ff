"""Parity of the multi-head latent attention path with the CPU oracle, through the C ABI:
the latent scoring store (576-dim rows, basis [M_lat 0; 0 I] of 128 rows), score + top-B with one
latent head (d 576, r 128, 64-token pages; one context past the sampling point, one ragged) and
the absorbed latent attention over the selected rows (32 query heads padded into one 128-head
tensor-core tile; 128 and 144 heads).
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
    def __init__(self, seq_lens, seed=1500):
        f = layer_factors(seed, 0, 1, D)
        qc, kc = sample_calibration(f, 2048, H_Q, seed)
        cal = O.calibrate(f64(qc)[..., :512], f64(kc)[..., :512], R_LAT)
        self.m_big = O.mla_scoring_basis(cal["M"][0]).astype(np.float32)[None]  # [1, 128, 576]
        kv = build_paged_kv(f, list(seq_lens), PS, seed, extra_pages=2)
        self.kv = kv["k_cache"]                      # [pages, 64, 1, 576]
        self.bt = kv["block_table"]
        self.lens_t = kv["seq_lens"]
        self.lens = np.asarray(seq_lens)
        self.q = sample_decode_queries(f, len(seq_lens), H_Q, seed)  # [batch, 32, 576]
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
    J.store(flat, slots, torch.from_numpy(case.m_big).cuda(), sc)
    assert check_codes(sc.cpu().numpy(), case.ys) <= 8


@pytest.mark.parametrize("budget", [2048, 700])
def test_mla_score_topk(case, budget):
    J = jssa()
    idx, count = J.score_topk(case.q.cuda(), torch.from_numpy(case.m_big).cuda(),
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
    idx, count = J.score_topk(c.q.cuda(), torch.from_numpy(c.m_big).cuda(),
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
