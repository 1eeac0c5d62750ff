"""Parity of the CUDA path (called through the C ABI) with the CPU oracle on seeded inputs.

Sizes: the tiny 2K-context workload (8 query / 2 KV heads, d 128, 16-token pages, r 32, B 128)
and variations that span several scan CTAs and ragged tails: uneven sequence lengths, lengths
below/at/above the budget, an empty sequence, r = 64, 32-token pages, contexts past the point
where the candidate threshold is sampled, candidate sets too large for shared staging, and an
adversarial score layout that defeats the sample.
Criteria are in ``parity.py``.
"""

import math

import numpy as np
import pytest
import torch

from oracle import jssa as O
from parity import (Case, check_codes, check_output, check_selection, f64)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from token_level_sparse_fp8_b200 import build
    build.build()


def jssa():
    import token_level_sparse_fp8_b200 as J
    return J


@pytest.fixture(scope="module")
def tiny():
    return Case([2048])


@pytest.fixture(scope="module")
def ragged():
    # lengths: long (several 1K-token CTAs), not a page multiple, just above / at / below the
    # budget, one token, empty
    return Case([2048, 1777, 129, 128, 127, 1, 0, 900], extra_pages=7, seed=1010)


def _select_oracle(case, budget):
    return O.select_step(case.np_q, case.m32.astype(np.float64), case.codes, case.np_bt,
                         case.np_lens, budget)


# ------------------------------------------------------------------------------------------------
# store
# ------------------------------------------------------------------------------------------------


@pytest.mark.parametrize("r", [16, 32, 64])
def test_store_codes(r):
    case = Case([2048, 300], r=r, seed=1020 + r)
    J = jssa()
    num_pages, ps, h_kv, d = case.k_cache.shape
    sc = torch.zeros((num_pages, h_kv, ps, r), dtype=torch.uint8, device="cuda")
    flat = case.gpu(case.k_cache).view(num_pages * ps, h_kv, d)
    slots = torch.arange(num_pages * ps, dtype=torch.int64, device="cuda")
    J.store(flat, slots, case.gpu_np(case.m32), sc)
    gpu = sc.cpu().numpy()
    n_mid = check_codes(gpu, case.ys)
    assert n_mid <= 2


def test_store_skips_negative_slots_and_partial_lists(tiny):
    J = jssa()
    num_pages, ps, h_kv, d = tiny.k_cache.shape
    sc = torch.full((num_pages, h_kv, ps, 32), 0xAB, dtype=torch.uint8, device="cuda")
    flat = tiny.gpu(tiny.k_cache).view(num_pages * ps, h_kv, d)
    slots = torch.arange(num_pages * ps, dtype=torch.int64, device="cuda")
    slots[::3] = -1
    J.store(flat, slots, tiny.gpu_np(tiny.m32), sc)
    gpu = sc.cpu().numpy().reshape(num_pages, h_kv, ps, 32).transpose(0, 2, 1, 3).reshape(-1, h_kv, 32)
    ref = tiny.codes.transpose(0, 2, 1, 3).reshape(-1, h_kv, 32)
    keep = np.ones(num_pages * ps, dtype=bool)
    keep[::3] = False
    assert np.all(gpu[~keep] == 0xAB)
    assert np.array_equal(gpu[keep], ref[keep])


# ------------------------------------------------------------------------------------------------
# score + top-B
# ------------------------------------------------------------------------------------------------


@pytest.mark.parametrize("budget", [1, 64, 128, 1000, 2047, 2048, 4096])
def test_score_topk_budgets(ragged, budget):
    J = jssa()
    idx, count = J.score_topk(ragged.gpu(ragged.q), ragged.gpu_np(ragged.m32),
                              ragged.gpu_np(ragged.codes), ragged.gpu(ragged.block_table),
                              ragged.gpu(ragged.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(ragged, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref_count)
    for b in range(len(ragged.seq_lens)):
        for h in range(ragged.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)


@pytest.mark.parametrize("seq_len,batch,budget", [(32768, 2, 2048), (20000, 1, 777), (65536, 1, 4096)])
def test_score_topk_long(seq_len, batch, budget):
    # contexts with a sampled candidate threshold, over many scan CTAs
    case = Case([seq_len] * batch, seed=1030 + seq_len % 97, calib=2048)
    J = jssa()
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(case.codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(case, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(batch):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)


def test_score_topk_rank64_and_page32():
    case = Case([3000, 1500], r=64, page_size=32, seed=1040)
    J = jssa()
    budget = 256
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(case.codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(case, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(2):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)


@pytest.mark.parametrize("page_size,lens,budget", [(16, [20000, 3000, 511], 512), (8, [17000, 900], 256)])
def test_score_topk_rank16(page_size, lens, budget):
    # 16-byte scoring rows: two 16-token tiles per warp copy instruction, a sampled threshold past
    # 16384 positions, a context under the budget; 8-token pages split a tile over two pages
    case = Case(lens, r=16, page_size=page_size, seed=1042 + page_size, calib=2048)
    J = jssa()
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(case.codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(case, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)


@pytest.mark.parametrize("page_size,lens,budget", [(4, [3000, 777], 200), (8, [20000], 512),
                                                     (8, [131072], 2048)])
def test_score_topk_small_pages(page_size, lens, budget):
    # pages shorter than a 16-token scan tile (rows of one tile come from several pages); the
    # 128K case takes 4096-position chunks, 256 candidate regions per pair (the flattened tier)
    case = Case(lens, page_size=page_size, seed=1045 + page_size, calib=2048)
    J = jssa()
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(case.codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(case, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for b in range(len(lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref_idx[b, h], ref_count[b, h], s[(b, h)], budget)


def test_score_topk_exact_ties_go_to_lower_position():
    # every token of a sequence gets the same code row -> all scores tie; the set must be the
    # lowest positions 0..B-1 on both sides
    case = Case([1500], seed=1050)
    codes = case.codes.copy()
    codes[:] = codes[0, :, :1, :]  # broadcast one row everywhere (per head)
    J = jssa()
    budget = 100
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    gi = idx.cpu().numpy()
    for h in range(case.h_kv):
        assert np.array_equal(gi[0, h], np.arange(budget))


def test_score_topk_long_ties_beyond_staging():
    # 40000 tied tokens: every key is a candidate (more than the select stage holds in shared
    # memory), and the set must still be the lowest positions
    case = Case([40000], seed=1051, calib=2048)
    codes = case.codes.copy()
    codes[:] = codes[0, :, :1, :]
    J = jssa()
    budget = 2048
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for h in range(case.h_kv):
        assert gc[0, h] == budget
        assert np.array_equal(gi[0, h], np.arange(budget))


def test_score_topk_budget_near_context():
    # a budget a third of the context: every position is a candidate, beyond shared staging
    case = Case([24000], seed=1052, calib=2048)
    J = jssa()
    budget = 8000
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(case.codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    ref_idx, ref_count, s = _select_oracle(case, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    for h in range(case.h_kv):
        check_selection(gi[0, h], gc[0, h], ref_idx[0, h], ref_count[0, h], s[(0, h)], budget)


def _mix32(x):
    x ^= x >> 16
    x = (x * 0x7FEB352D) & 0xFFFFFFFF
    x ^= x >> 15
    x = (x * 0x846CA68B) & 0xFFFFFFFF
    x ^= x >> 16
    return x


def _sampled_positions(pair, L, groups=512, run=4):
    # the candidate-threshold sample of the score kernels: one run of 4 consecutive positions per
    # stratum of L // 512 tokens, starting at a 4-aligned offset drawn from a 32-bit mix of
    # (stratum, pair) scaled to the stratum by a high multiply
    stratum = L // groups
    out = []
    for g in range(groups):
        h = _mix32(((g * 0x9E3779B9) & 0xFFFFFFFF) ^ ((pair * 0x85EBCA6B + 1) & 0xFFFFFFFF))
        first = (g * stratum + run - 1) // run
        p0 = run * (first + ((h * (stratum // run - 1)) >> 32))
        out.extend(range(p0, p0 + run))
    return np.asarray(out)


def test_score_topk_rescan_when_sample_overestimates():
    # adversarial scores: exactly the sampled positions score high, every other position low, so
    # the sampled threshold lets through 2048 keys for a budget of 4096; the selection must detect
    # it, rescan the sequence and still return the exact set (and say so in the device flags)
    L, budget = 32768, 4096
    case = Case([L], seed=1053, calib=2048)
    codes = case.codes.copy()
    bt = case.np_bt
    qbar = O.group_mean_query(case.np_q[0], case.h_kv)
    for h in range(case.h_kv):
        row = codes[bt[0, 0], h, 0, :].copy()
        s0 = O.scores(row[None, :], O.projected_query(qbar[h], case.m32[h].astype(np.float64)))[0]
        assert s0 != 0.0
        hi, lo = (row, row ^ 0x80) if s0 > 0 else (row ^ 0x80, row)
        sampled = np.zeros(L, dtype=bool)
        sampled[_sampled_positions(h, L)] = True
        for pos in range(L):
            codes[bt[0, pos // case.ps], h, pos % case.ps, :] = hi if sampled[pos] else lo
    J = jssa()
    J.device_error(clear=True)
    idx, count = J.score_topk(case.gpu(case.q), case.gpu_np(case.m32), case.gpu_np(codes),
                              case.gpu(case.block_table), case.gpu(case.seq_lens_t), budget)
    flags = J.device_error(clear=True)
    ref_idx, ref_count, _ = O.select_step(case.np_q, case.m32.astype(np.float64), codes, bt,
                                          case.np_lens, budget)
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref_count)
    assert np.array_equal(gi, ref_idx)
    assert flags == 16


# ------------------------------------------------------------------------------------------------
# attention
# ------------------------------------------------------------------------------------------------


def test_indexed_attend_on_oracle_sets(ragged):
    J = jssa()
    budget = 128
    ref_idx, ref_count, _ = _select_oracle(ragged, budget)
    scale = 1.0 / math.sqrt(ragged.d)
    out = J.indexed_attend(ragged.gpu(ragged.q), ragged.gpu(ragged.k_cache),
                           ragged.gpu(ragged.v_cache), ragged.gpu(ragged.block_table),
                           ragged.gpu_np(ref_idx), ragged.gpu_np(ref_count), scale)
    ref = O.indexed_attend_step(ragged.np_q, ragged.np_k, ragged.np_v, ragged.np_bt, ref_idx,
                                ref_count, scale)
    check_output(f64(out), ref)
    # the empty sequence gives zeros
    assert torch.count_nonzero(out[6]).item() == 0


def test_indexed_attend_long_sets_many_splits():
    case = Case([6000, 4100], seed=1060, calib=2048)
    J = jssa()
    budget = 4096
    ref_idx, ref_count, _ = _select_oracle(case, budget)
    scale = 0.3
    ws = J.Workspace("cuda")
    args = (case.gpu(case.q), case.gpu(case.k_cache), case.gpu(case.v_cache),
            case.gpu(case.block_table), case.gpu_np(ref_idx), case.gpu_np(ref_count), scale)
    out1 = J.indexed_attend(*args, ws=ws)
    out2 = J.indexed_attend(*args, ws=ws)  # the tickets were reset by the first call
    ref = O.indexed_attend_step(case.np_q, case.np_k, case.np_v, case.np_bt, ref_idx, ref_count, scale)
    check_output(f64(out1), ref)
    assert torch.equal(out1, out2)


@pytest.mark.parametrize("window", [-1, 100, 1024])
def test_dense_decode(ragged, window):
    J = jssa()
    scale = 1.0 / math.sqrt(ragged.d)
    out = J.dense_decode(ragged.gpu(ragged.q), ragged.gpu(ragged.k_cache),
                         ragged.gpu(ragged.v_cache), ragged.gpu(ragged.block_table),
                         ragged.gpu(ragged.seq_lens_t), scale, window)
    ref = O.dense_step(ragged.np_q, ragged.np_k, ragged.np_v, ragged.np_bt, ragged.np_lens, scale,
                       window)
    check_output(f64(out), ref)


def test_dense_equals_full_budget_jssa(tiny):
    # B >= L: the sparse step attends to every position, so it must agree with dense attention
    J = jssa()
    layer = J.PagedLayer(tiny.gpu(tiny.k_cache), tiny.gpu(tiny.v_cache), tiny.gpu(tiny.block_table),
                         tiny.gpu(tiny.seq_lens_t), tiny.gpu_np(tiny.m32), budget=4096)
    layer.prefill_scores()
    q = tiny.gpu(tiny.q)
    out, idx, count = layer.step(q)
    dense = layer.dense(q)
    assert count.cpu().numpy().tolist() == [[2048, 2048]]
    check_output(f64(out), f64(dense))


# ------------------------------------------------------------------------------------------------
# whole decode step
# ------------------------------------------------------------------------------------------------


@pytest.mark.parametrize("budget", [128, 700])
def test_decode_step(ragged, budget):
    J = jssa()
    case = ragged
    lens = np.asarray(case.seq_lens)
    rng = np.random.default_rng(5)
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
    # caches: the new rows and codes were written at position L-1 of every live sequence
    assert np.array_equal(f64(k_cache), ref["k_cache"])
    assert np.array_equal(f64(v_cache), ref["v_cache"])
    gsc = sc.cpu().numpy()
    assert np.array_equal(gsc, ref["score_cache"])
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref["count"])
    for b in range(len(lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref["idx"][b, h], ref["count"][b, h],
                            ref["scores"][(b, h)], budget)
    check_output(f64(out), ref["out"])


@pytest.mark.parametrize("h_q,h_kv,lens,budget", [(8, 1, [20000, 3000], 512),  # MQA, G = 8
                                                   (4, 4, [5000, 700], 256)])     # G = 1
def test_decode_step_group_sizes(h_q, h_kv, lens, budget):
    # the largest group the attention's m16 tile holds (8 query heads on one KV head) and one query
    # head per KV head, through the whole decode step with a new token
    J = jssa()
    case = Case(lens, h_q=h_q, h_kv=h_kv, seed=1090 + h_q * 10 + h_kv, calib=2048)
    rng = np.random.default_rng(9)
    k_new = torch.from_numpy(rng.standard_normal((len(lens), h_kv, case.d))).to(torch.bfloat16)
    v_new = torch.from_numpy(rng.standard_normal((len(lens), h_kv, case.d))).to(torch.bfloat16)
    k_cache, v_cache = case.gpu(case.k_cache).clone(), case.gpu(case.v_cache).clone()
    sc = case.gpu_np(case.codes).clone()
    scale = 1.0 / math.sqrt(case.d)
    out, idx, count = J.decode(case.gpu(case.q), k_new.cuda(), v_new.cuda(), k_cache, v_cache, sc,
                               case.gpu_np(case.m32), case.gpu(case.block_table),
                               case.gpu(case.seq_lens_t), budget, scale)
    ref = O.decode_step(case.np_q, f64(k_new), f64(v_new), case.np_k, case.np_v, case.codes,
                        case.np_bt, np.asarray(lens), case.m32.astype(np.float64), budget, scale)
    assert np.array_equal(sc.cpu().numpy(), ref["score_cache"])
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref["count"])
    for b in range(len(lens)):
        for h in range(h_kv):
            check_selection(gi[b, h], gc[b, h], ref["idx"][b, h], ref["count"][b, h],
                            ref["scores"][(b, h)], budget)
    check_output(f64(out), ref["out"])


@pytest.mark.parametrize("page_size,lens,budget", [(64, [20000, 1000], 512), (128, [17001, 300], 256)])
def test_decode_step_large_pages(page_size, lens, budget):
    # pages larger than a scan chunk's 16-token tiles and than an attention tile: several tiles and
    # several selected rows per page, the new token in the middle of its page
    J = jssa()
    case = Case(lens, page_size=page_size, seed=1100 + page_size, calib=2048)
    rng = np.random.default_rng(11)
    k_new = torch.from_numpy(rng.standard_normal((len(lens), case.h_kv, case.d))).to(torch.bfloat16)
    v_new = torch.from_numpy(rng.standard_normal((len(lens), case.h_kv, case.d))).to(torch.bfloat16)
    k_cache, v_cache = case.gpu(case.k_cache).clone(), case.gpu(case.v_cache).clone()
    sc = case.gpu_np(case.codes).clone()
    scale = 1.0 / math.sqrt(case.d)
    out, idx, count = J.decode(case.gpu(case.q), k_new.cuda(), v_new.cuda(), k_cache, v_cache, sc,
                               case.gpu_np(case.m32), case.gpu(case.block_table),
                               case.gpu(case.seq_lens_t), budget, scale)
    ref = O.decode_step(case.np_q, f64(k_new), f64(v_new), case.np_k, case.np_v, case.codes,
                        case.np_bt, np.asarray(lens), case.m32.astype(np.float64), budget, scale)
    assert np.array_equal(f64(k_cache), ref["k_cache"])
    assert np.array_equal(sc.cpu().numpy(), ref["score_cache"])
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref["count"])
    for b in range(len(lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref["idx"][b, h], ref["count"][b, h],
                            ref["scores"][(b, h)], budget)
    check_output(f64(out), ref["out"])


def test_decode_step_is_deterministic(ragged):
    # the same step on the same inputs gives bit-identical outputs, index sets and caches (the
    # split-K merge combines the splits in a fixed order whichever CTA finishes last)
    J = jssa()
    case = ragged
    rng = np.random.default_rng(13)
    k_new = torch.from_numpy(rng.standard_normal((len(case.seq_lens), case.h_kv, case.d))).to(torch.bfloat16).cuda()
    v_new = torch.from_numpy(rng.standard_normal((len(case.seq_lens), case.h_kv, case.d))).to(torch.bfloat16).cuda()
    results = []
    for _ in range(2):
        k_cache, v_cache = case.gpu(case.k_cache).clone(), case.gpu(case.v_cache).clone()
        sc = case.gpu_np(case.codes).clone()
        out, idx, count = J.decode(case.gpu(case.q), k_new, v_new, k_cache, v_cache, sc,
                                   case.gpu_np(case.m32), case.gpu(case.block_table),
                                   case.gpu(case.seq_lens_t), 700, 1.0 / math.sqrt(case.d))
        results.append((out.cpu(), idx.cpu(), count.cpu(), sc.cpu(), k_cache.cpu()))
    for a, b in zip(*results):
        assert torch.equal(a, b)


def test_decode_step_long_contexts():
    # contexts past the all-candidates limit: the new token is stored by the same kernel that
    # draws the threshold sample, and the scan reads its code afterwards
    case = Case([20000, 17001, 16384], seed=1070, calib=2048)
    J = jssa()
    budget = 1024
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
    assert np.array_equal(sc.cpu().numpy(), ref["score_cache"])
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref["count"])
    for b in range(len(lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref["idx"][b, h], ref["count"][b, h],
                            ref["scores"][(b, h)], budget)
    check_output(f64(out), ref["out"])


def test_decode_step_rank16():
    # the fused decode store and the whole step at r = 16
    case = Case([20000, 5000, 96], r=16, seed=1075, calib=2048)
    J = jssa()
    budget = 512
    lens = np.asarray(case.seq_lens)
    rng = np.random.default_rng(9)
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
    assert np.array_equal(sc.cpu().numpy(), ref["score_cache"])
    gi, gc = idx.cpu().numpy(), count.cpu().numpy()
    assert np.array_equal(gc, ref["count"])
    for b in range(len(lens)):
        for h in range(case.h_kv):
            check_selection(gi[b, h], gc[b, h], ref["idx"][b, h], ref["count"][b, h],
                            ref["scores"][(b, h)], budget)
    check_output(f64(out), ref["out"])


def test_page_permutation_invariance_on_gpu(tiny):
    # the same logical cache under another physical page order gives identical results
    J = jssa()
    num_pages = tiny.k_cache.shape[0]
    remap = torch.arange(num_pages - 1, -1, -1)
    inv = torch.argsort(remap)
    bt2 = remap[tiny.block_table.long()].to(torch.int32)
    args1 = (tiny.gpu(tiny.k_cache), tiny.gpu(tiny.v_cache), tiny.gpu_np(tiny.codes), tiny.gpu(tiny.block_table))
    args2 = (tiny.gpu(tiny.k_cache[inv]), tiny.gpu(tiny.v_cache[inv]),
             tiny.gpu_np(tiny.codes[inv.numpy()]), tiny.gpu(bt2))
    res = []
    for kc, vc, sc, bt in (args1, args2):
        res.append(J.decode(tiny.gpu(tiny.q), None, None, kc, vc, sc, tiny.gpu_np(tiny.m32), bt,
                            tiny.gpu(tiny.seq_lens_t), 128, 0.1))
    assert torch.equal(res[0][1], res[1][1])
    assert torch.equal(res[0][0], res[1][0])


def test_device_flags_for_corrupt_page_table(tiny):
    J = jssa()
    J.device_error(clear=True)
    bt = tiny.block_table.clone()
    bt[0, 5] = 10_000_000  # page beyond the pool
    bt[0, 9] = -3
    out, idx, count = J.decode(tiny.gpu(tiny.q), None, None, tiny.gpu(tiny.k_cache),
                               tiny.gpu(tiny.v_cache), tiny.gpu_np(tiny.codes),
                               tiny.gpu_np(tiny.m32), tiny.gpu(bt), tiny.gpu(tiny.seq_lens_t), 128,
                               0.1)
    flags = J.device_error(clear=True)
    assert flags & 1
    assert torch.isfinite(out.float()).all()
    assert J.device_error(clear=True) == 0


# ------------------------------------------------------------------------------------------------
# calibration
# ------------------------------------------------------------------------------------------------


@pytest.mark.parametrize("n", [4096, 1000])
def test_calibration(tiny, n):
    from synth import sample_calibration
    J = jssa()
    q, k = sample_calibration(tiny.factors, n, tiny.h_q // tiny.h_kv, tiny.seed)
    res = O.calibrate(f64(q), f64(k), tiny.r)
    got = J.calibrate(q.cuda(), k.cuda(), tiny.r, batch=1536)
    gq, gk = f64(got["gram_q"]), f64(got["gram_k"])
    for g, rg in ((gq, res["gram_q"]), (gk, res["gram_k"])):
        assert np.max(np.abs(g - rg)) <= 1e-5 * np.max(np.abs(rg))
    m = f64(got["M"])
    lam = f64(got["eigvals"])
    for h in range(tiny.h_kv):
        assert np.max(np.abs(m[h] @ m[h].T - np.eye(tiny.r))) <= 1e-6
        p_gpu, p_ref = O.projector(m[h]), O.projector(res["M"][h])
        assert np.max(np.abs(p_gpu - p_ref)) <= 1e-4
        a_q, a_k = O.unit_trace(res["gram_q"][h]), O.unit_trace(res["gram_k"][h])
        opt = O.l_marg(p_ref, a_q, a_k)
        assert -1e-9 <= O.l_marg(p_gpu, a_q, a_k) - opt <= 1e-7
        assert np.max(np.abs(lam[h] - res["eigvals"][h])) <= 1e-5 * lam[h, 0]
        # rows agree with the oracle's rows up to the shared sign rule
        assert np.max(np.abs(m[h] - res["M"][h])) <= 5e-3


def test_calibration_many_heads_per_group():
    # 32 query heads per KV head (G d = 4096): the Gram kernel forms the group mean and sums its
    # bf16 planes instead of the G^2 head products
    from synth import layer_factors, sample_calibration
    J = jssa()
    h_kv, d, g, r = 2, 128, 32, 32
    f = layer_factors(1530, 0, h_kv, d)
    q, k = sample_calibration(f, 1000, g, 1530)
    res = O.calibrate(f64(q), f64(k), r)
    got = J.calibrate(q.cuda(), k.cuda(), r, batch=700)
    for gg, rg in ((f64(got["gram_q"]), res["gram_q"]), (f64(got["gram_k"]), res["gram_k"])):
        assert np.max(np.abs(gg - rg)) <= 1e-5 * np.max(np.abs(rg))
    m = f64(got["M"])
    for h in range(h_kv):
        a_q, a_k = O.unit_trace(res["gram_q"][h]), O.unit_trace(res["gram_k"][h])
        opt = O.l_marg(O.projector(res["M"][h]), a_q, a_k)
        basis64, _ = np.linalg.qr(m[h].T)  # the float32 rows' subspace as an exact projector
        assert -1e-12 <= O.l_marg(basis64 @ basis64.T, a_q, a_k) - opt <= 1e-7


# ------------------------------------------------------------------------------------------------
# gather-then-attend (the ablation the gather-free attention is compared with)
# ------------------------------------------------------------------------------------------------


def test_gather_kv_is_an_exact_copy(ragged):
    J = jssa()
    budget = 128
    ref_idx, ref_count, _ = _select_oracle(ragged, budget)
    k, v, lens = J.gather_kv(ragged.gpu(ragged.k_cache), ragged.gpu(ragged.v_cache),
                             ragged.gpu(ragged.block_table), ragged.gpu_np(ref_idx),
                             ragged.gpu_np(ref_count))
    assert lens.cpu().numpy().tolist() == ref_count[:, 0].tolist()
    kc, vc = ragged.k_cache.view(torch.int16).numpy(), ragged.v_cache.view(torch.int16).numpy()
    gk, gv = k.cpu().view(torch.int16).numpy(), v.cpu().view(torch.int16).numpy()
    ps = ragged.ps
    for b in range(len(ragged.seq_lens)):
        for h in range(ragged.h_kv):
            for j in range(ref_count[b, h]):
                t = ref_idx[b, h, j]
                page = ragged.np_bt[b, t // ps]
                assert np.array_equal(gk[b, j, h], kc[page, t % ps, h])
                assert np.array_equal(gv[b, j, h], vc[page, t % ps, h])


@pytest.mark.parametrize("budget", [128, 1000])
def test_gather_then_attend(ragged, budget):
    J = jssa()
    ref_idx, ref_count, _ = _select_oracle(ragged, budget)
    scale = 1.0 / math.sqrt(ragged.d)
    out = J.gather_then_attend(ragged.gpu(ragged.q), ragged.gpu(ragged.k_cache),
                               ragged.gpu(ragged.v_cache), ragged.gpu(ragged.block_table),
                               ragged.gpu_np(ref_idx), ragged.gpu_np(ref_count), scale)
    ref = O.indexed_attend_step(ragged.np_q, ragged.np_k, ragged.np_v, ragged.np_bt, ref_idx,
                                ref_count, scale)
    check_output(f64(out), ref)
    gf = J.indexed_attend(ragged.gpu(ragged.q), ragged.gpu(ragged.k_cache),
                          ragged.gpu(ragged.v_cache), ragged.gpu(ragged.block_table),
                          ragged.gpu_np(ref_idx), ragged.gpu_np(ref_count), scale)
    check_output(f64(gf), ref)
