"""The allocation-free indexed attention (``jssa_indexed_attend_noalloc``) against the regular
entry point (``jssa_indexed_attend``), both called through the C ABI.

The allocation-free variant exists for callers that cannot provide device memory of their own
(a runtime that owns all device memory and gives plug-ins no allocator, a loop that must not
call cudaMalloc and its implicit device synchronisation, a host program that only links the C
ABI). It keeps its split-K scratch in a fixed device array inside the library instead of a
workspace. Two calls in a row must both agree with the regular entry point within the parity
tolerance; the second call also shows that the scratch left behind by the first (ticket counters
and partials) does not leak into the next result.

This file is collected last on purpose, so that a stop-at-first-failure run has already run every
other test when it gets here; it builds its own inputs and also passes alone in a fresh process.
"""

import ctypes
import math

import numpy as np
import pytest
import torch

from oracle import jssa as O
from parity import Case, check_output, f64

pytestmark = pytest.mark.gpu


def _raw(t):
    return t.data_ptr()


def test_noalloc_matches_regular_entry_point_twice():
    from token_level_sparse_fp8_b200 import _lib, build, api
    build.build()
    lib = _lib.load()
    case = Case([2048, 1300, 700, 96, 0], seed=1090, extra_pages=4)
    budget = 512
    ref_idx, ref_count, _ = O.select_step(case.np_q, case.m32.astype(np.float64), case.codes,
                                          case.np_bt, case.np_lens, budget)
    dev = torch.device("cuda")
    q = case.q.to(dev)
    k_cache, v_cache = case.k_cache.to(dev), case.v_cache.to(dev)
    bt = case.block_table.to(dev)
    idx = torch.from_numpy(ref_idx).to(dev)
    count = torch.from_numpy(ref_count).to(dev)
    batch, h_q, d = q.shape
    num_pages, page_size, h_kv, _ = k_cache.shape
    ps, ss, hs = api.kv_strides(k_cache)
    scale = 1.0 / math.sqrt(d)
    stream = torch.cuda.current_stream(dev).cuda_stream

    # the regular entry point with a caller-provided workspace
    nbytes = api.workspace_size(_lib.FN_INDEXED_ATTEND, batch, h_q, h_kv, d, bt.shape[1], page_size,
                                budget)
    assert 0 < nbytes <= 4 << 20
    ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
    out_ref = torch.empty_like(q)
    st = lib.jssa_indexed_attend(_raw(q), _raw(k_cache), _raw(v_cache), ps, ss, hs, _raw(bt),
                                 bt.shape[1], _raw(idx), _raw(count), batch, h_q, h_kv, d, budget,
                                 num_pages, page_size, ctypes.c_float(scale), _raw(out_ref),
                                 _raw(ws), nbytes, stream)
    assert st == 0, _lib.status_string(st)

    outs = []
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        st = lib.jssa_indexed_attend_noalloc(_raw(q), _raw(k_cache), _raw(v_cache), ps, ss, hs,
                                             _raw(bt), bt.shape[1], _raw(idx), _raw(count), batch,
                                             h_q, h_kv, d, budget, num_pages, page_size,
                                             ctypes.c_float(scale), _raw(out), stream)
        assert st == 0, _lib.status_string(st)
        outs.append(out)
    torch.cuda.synchronize(dev)
    ref = f64(out_ref)
    for out in outs:
        got = f64(out)
        assert np.isfinite(got).all()
        check_output(got, ref)
    # and both stay within the oracle's tolerance
    oracle = O.indexed_attend_step(case.np_q, case.np_k, case.np_v, case.np_bt, ref_idx, ref_count, scale)
    check_output(f64(outs[1]), oracle)
