"""Parity of the bf16 scoring-cache ablation (jssa_store_bf16, jssa_score_topk_bf16) with the
CPU oracle: the cache holds bf16(M k) (one rounding of the float64 product), the scores multiply
those values by p. Sizes: several scan CTAs, the sampled candidate threshold (a context past
16384 tokens) and a ragged one. Criteria are in ``parity.py``.
"""

import numpy as np
import pytest
import torch

from oracle import jssa as O
from oracle.bf16 import bf16_decode, bf16_encode
from parity import Case, check_selection

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from token_level_sparse_fp8_b200 import build
    build.build()


def jssa():
    import token_level_sparse_fp8_b200 as J
    return J


def bf16_cache(case):
    """Oracle bf16 codes ``uint16 [pages, h_kv, ps, r]`` and the float64 projections."""
    num_pages, ps, h_kv, d = case.np_k.shape
    codes = np.zeros((num_pages, h_kv, ps, case.r), dtype=np.uint16)
    ys = np.zeros((num_pages, h_kv, ps, case.r))
    for h in range(h_kv):
        y = case.np_k[:, :, h].reshape(-1, d) @ case.m32[h].astype(np.float64).T
        ys[:, h] = y.reshape(num_pages, ps, case.r)
        codes[:, h] = O.store_codes_bf16(case.np_k[:, :, h].reshape(-1, d),
                                         case.m32[h]).reshape(num_pages, ps, case.r)
    return codes, ys


@pytest.fixture(scope="module")
def case():
    c = Case([20000, 3000], seed=1400, calib=2048)
    c.bf16_codes, c.bf16_ys = bf16_cache(c)
    return c


def test_bf16_store_codes(case):
    J = jssa()
    num_pages, ps, h_kv, d = case.k_cache.shape
    sc = torch.zeros((num_pages, h_kv, ps, case.r), dtype=torch.bfloat16, device="cuda")
    flat = case.gpu(case.k_cache).view(num_pages * ps, h_kv, d)
    slots = torch.arange(num_pages * ps, dtype=torch.int64, device="cuda")
    J.store(flat, slots, case.gpu_np(case.m32), sc)
    got = sc.cpu().view(torch.int16).numpy().view(np.uint16)
    ref = case.bf16_codes
    diff = got != ref
    if diff.any():
        # allowed only where the float64 projection sits on a rounding midpoint to within the
        # difference of two float64 summation orders
        a, b = bf16_decode(got[diff]), bf16_decode(ref[diff])
        y = case.bf16_ys[diff]
        assert np.all(np.abs(y - 0.5 * (a + b)) <= 1e-12 * np.abs(y)), "codes differ off a midpoint"
        assert diff.sum() <= 4


@pytest.mark.parametrize("budget", [2048, 300])
def test_bf16_score_topk(case, budget):
    J = jssa()
    sc = torch.from_numpy(case.bf16_codes.view(np.int16)).view(torch.bfloat16).cuda()
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), sc,
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    ref_idx, ref_count, s = O.select_step(case.np_q, case.m32.astype(np.float64), case.bf16_codes,
                                          case.np_bt, case.np_lens, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(case.seq_lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)


def test_bf16_score_topk_small_pages_and_short():
    J = jssa()
    c = Case([17000, 200, 0], page_size=4, seed=1410, calib=1024, extra_pages=3)
    codes, _ = bf16_cache(c)
    budget = 256
    sc = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).cuda()
    idx, count = J.score_topk(c.gpu(c.q), c.gpu_np(c.m32), sc, c.gpu(c.block_table),
                              c.gpu(c.seq_lens_t), budget)
    ref_idx, ref_count, s = O.select_step(c.np_q, c.m32.astype(np.float64), codes, c.np_bt,
                                          c.np_lens, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(c.seq_lens)):
        for h in range(c.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)
