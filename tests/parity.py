"""Parity criteria between the CUDA path and the CPU oracle, and case builders for the tests.

Tolerances (stated once, used by every parity test):
* page-table, index and count handling: bit-exact;
* FP8 scoring codes: bit-exact, except a one-step difference where the oracle's float64
  projection lies within a relative 1e-6 of the rounding midpoint between the two codes;
* index sets: equal sizes; a position may be in one set and not the other only if its oracle
  score is within 1e-4 * max|score| of the oracle's budget-th largest score (ties go to the lower
  position on both sides);
* attention outputs (bf16): max-abs error <= 1e-2 and mean relative error
  sum|gpu - oracle| / sum|oracle| <= 2e-3 against the float64 oracle.
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import jssa as O
from oracle.fp8 import e4m3_decode, e4m3_encode
from synth import build_paged_kv, layer_factors, sample_calibration, sample_decode_queries

CODE_MIDPOINT_REL = 1e-6
SCORE_TIE_REL = 1e-4
OUT_MAX_ABS = 1e-2
OUT_MEAN_REL = 2e-3


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def check_codes(gpu_codes: np.ndarray, y: np.ndarray) -> int:
    """Codes vs the oracle's float64 projections ``y``; returns the number of tolerated
    midpoint differences."""
    ref = e4m3_encode(y)
    diff = gpu_codes != ref
    if not diff.any():
        return 0
    a = e4m3_decode(gpu_codes[diff])
    b = e4m3_decode(ref[diff])
    yd = y[diff]
    mid = 0.5 * (a + b)
    ok = np.abs(yd - mid) <= CODE_MIDPOINT_REL * np.maximum(np.abs(yd), 1e-30)
    # the two codes must be neighbours (one rounding step apart)
    step = np.abs(gpu_codes[diff].astype(np.int64) - ref[diff].astype(np.int64))
    assert np.all(ok & (step == 1)), (
        f"{(~ok).sum()} codes differ away from a rounding midpoint: y={yd[~ok][:5]}, "
        f"gpu={a[~ok][:5]}, oracle={b[~ok][:5]}")
    return int(diff.sum())


def check_selection(gpu_idx: np.ndarray, gpu_count: int, ref_idx: np.ndarray, ref_count: int,
                    s: np.ndarray, budget: int) -> int:
    """One (sequence, KV head) index set; returns the number of tolerated near-tie swaps."""
    L = s.shape[0]
    assert gpu_count == ref_count == min(budget, L)
    g = gpu_idx[:gpu_count]
    assert np.all(gpu_idx[gpu_count:] == -1), "padding must be -1"
    assert np.all(np.diff(g) > 0), "index set must be strictly ascending"
    if gpu_count:
        assert g[0] >= 0 and g[-1] < L
    sym = np.setxor1d(g, ref_idx[:ref_count])
    if sym.size:
        kth = np.sort(s)[::-1][min(budget, L) - 1]
        tol = SCORE_TIE_REL * np.max(np.abs(s))
        bad = sym[np.abs(s[sym] - kth) > tol]
        assert bad.size == 0, f"positions {bad[:8]} differ by more than the tie tolerance"
    return int(sym.size // 2)


def check_output(gpu: np.ndarray, ref: np.ndarray) -> dict:
    err = np.abs(gpu - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.abs(ref).sum())
    mean_rel = float(err.sum() / denom) if denom > 0 else float(err.sum())
    assert max_abs <= OUT_MAX_ABS, f"max-abs error {max_abs}"
    assert mean_rel <= OUT_MEAN_REL, f"mean relative error {mean_rel}"
    return {"max_abs": max_abs, "mean_rel": mean_rel}


def oracle_basis(seed: int, h_kv: int, h_q: int, d: int, r: int, n: int, factors=None):
    """The oracle's calibration on the generator's samples, rounded to float32 (the basis both
    sides then use)."""
    f = factors or layer_factors(seed, 0, h_kv, d)
    q, k = sample_calibration(f, n, h_q // h_kv, seed)
    res = O.calibrate(f64(q), f64(k), r)
    return res["M"].astype(np.float32), res


def oracle_score_cache(k_cache: np.ndarray, m32: np.ndarray):
    """Oracle store of every slot: codes ``uint8 [pages, h_kv, ps, r]`` and the float64
    projections."""
    num_pages, ps, h_kv, d = k_cache.shape
    r = m32.shape[1]
    codes = np.zeros((num_pages, h_kv, ps, r), dtype=np.uint8)
    ys = np.zeros((num_pages, h_kv, ps, r))
    for h in range(h_kv):
        y = k_cache[:, :, h].reshape(-1, d) @ m32[h].astype(np.float64).T
        ys[:, h] = y.reshape(num_pages, ps, r)
        codes[:, h] = e4m3_encode(y).reshape(num_pages, ps, r)
    return codes, ys


class Case:
    """A small decode workload built on the CPU (generator) and mirrored on the GPU."""

    def __init__(self, seq_lens, h_q=8, h_kv=2, d=128, r=32, page_size=16, seed=1000,
                 calib=4096, extra_pages=5, device="cuda"):
        self.seq_lens = list(seq_lens)
        self.h_q, self.h_kv, self.d, self.r, self.ps = h_q, h_kv, d, r, page_size
        f = layer_factors(seed, 0, h_kv, d)
        self.m32, self.calib = oracle_basis(seed, h_kv, h_q, d, r, calib, factors=f)
        kv = build_paged_kv(f, self.seq_lens, page_size, seed, extra_pages=extra_pages)
        self.k_cache = kv["k_cache"]
        self.v_cache = kv["v_cache"]
        self.block_table = kv["block_table"]
        self.seq_lens_t = kv["seq_lens"]
        self.q = sample_decode_queries(f, len(self.seq_lens), h_q // h_kv, seed)
        self.factors = f
        self.seed = seed
        self.dev = torch.device(device)
        # numpy views for the oracle
        self.np_k = f64(self.k_cache)
        self.np_v = f64(self.v_cache)
        self.np_q = f64(self.q)
        self.np_bt = self.block_table.numpy()
        self.np_lens = np.asarray(self.seq_lens)
        self.codes, self.ys = oracle_score_cache(self.np_k, self.m32)

    def gpu(self, t: torch.Tensor) -> torch.Tensor:
        return t.to(self.dev)

    def gpu_np(self, a: np.ndarray) -> torch.Tensor:
        return torch.from_numpy(np.ascontiguousarray(a)).to(self.dev)
