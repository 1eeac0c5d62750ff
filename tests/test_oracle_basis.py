"""Pins of the oracle's calibration (joint basis) against the mathematics the pages state.

* ``M M^T = I_r`` (JSSA summary, Theoretical Foundation: orthonormal basis);
* Ky Fan: the minimum of ``L_marg`` over rank-r projectors is ``tr A - sum of the r largest
  eigenvalues = 2 - sum_{i<=r} lambda_i`` (unit traces), reached by eq. (5);
* brute force over random projectors (and a grid of directions) for d in {3, 4}: none beats
  eq. (5) on ``L_marg`` (eqs. (4)-(5));
* the bound of eq. (4), ``L_sel <= 1/4 L_marg^2``, on random projectors of every rank, through
  the intermediate product ``tr((I-P)A_Q) tr((I-P)A_K)``;
* scale invariance of each second moment (unit-trace normalisation, eq. (3));
* LAPACK ``eigh`` against the independent Jacobi solver in ``oracle.jacobi``;
* planted mistakes (ascending eigen-order, no normalisation) are caught by these pins.
"""

import numpy as np
import pytest
import torch

from oracle import jssa as O
from oracle.jacobi import jacobi_eigh
from synth import WORKLOADS, layer_factors, sample_calibration


def _rand_psd(rng, d, rank=None):
    x = rng.standard_normal((d, rank or d))
    a = x @ x.T
    return a / np.trace(a)


def _rand_projectors(rng, n, d, r):
    q, _ = np.linalg.qr(rng.standard_normal((n, d, r)))
    return np.swapaxes(q, -1, -2)  # [n, r, d] orthonormal rows


def _lmarg_batch(m, a):
    # tr((I - P) A) = tr A - sum_k m_k^T A m_k for orthonormal rows m_k
    return np.trace(a) - np.einsum("nkd,de,nke->n", m, a, m)


@pytest.fixture(scope="module")
def tiny_calib():
    w = WORKLOADS["tiny"]
    f = layer_factors(w.seed, 0, w.h_kv, w.d)
    q, k = sample_calibration(f, w.calib_samples, w.group, w.seed)
    res = O.calibrate(q.to(torch.float64).numpy(), k.to(torch.float64).numpy(), w.rank)
    return w, res


def test_basis_orthonormal(tiny_calib):
    w, res = tiny_calib
    m = res["M"]
    assert m.shape == (w.h_kv, w.rank, w.d)
    for h in range(w.h_kv):
        assert np.max(np.abs(m[h] @ m[h].T - np.eye(w.rank))) <= 1e-12


def test_ky_fan_closed_form(tiny_calib):
    w, res = tiny_calib
    for h in range(w.h_kv):
        a_q = O.unit_trace(res["gram_q"][h])
        a_k = O.unit_trace(res["gram_k"][h])
        lam = res["eigvals"][h]
        assert abs(np.sum(lam) - 2.0) <= 1e-12
        assert np.all(np.diff(lam) <= 1e-15)
        p = O.projector(res["M"][h])
        assert abs(O.l_marg(p, a_q, a_k) - (2.0 - lam[: w.rank].sum())) <= 1e-12


def test_spectral_gap_of_generator(tiny_calib):
    # The projector is unique only when lambda_r > lambda_{r+1}; the generator keeps a gap.
    w, res = tiny_calib
    lam = res["eigvals"]
    gap = (lam[:, w.rank - 1] - lam[:, w.rank]) / lam[:, w.rank - 1]
    assert np.all(gap > 1e-3)


@pytest.mark.parametrize("d,r", [(3, 1), (3, 2), (4, 1), (4, 2)])
def test_bruteforce_projectors_never_beat_topeig(d, r):
    rng = np.random.default_rng(100 + 10 * d + r)
    for trial in range(5):
        a_q = _rand_psd(rng, d, rank=rng.integers(1, d + 1))
        a_k = _rand_psd(rng, d, rank=rng.integers(1, d + 1))
        m_star, _ = O.joint_basis(a_q[None], a_k[None], r)
        best = O.l_marg(O.projector(m_star[0]), a_q, a_k)
        cand = _rand_projectors(rng, 100_000, d, r)
        vals = _lmarg_batch(cand, a_q + a_k)
        assert vals.min() >= best - 1e-12
        # and the search gets close, so the optimum is really attained there
        assert vals.min() - best <= 5e-2
    if d == 3 and r == 1:
        # a deterministic grid of unit directions on the sphere
        th, ph = np.meshgrid(np.linspace(0, np.pi, 181), np.linspace(0, 2 * np.pi, 361))
        dirs = np.stack([np.sin(th) * np.cos(ph), np.sin(th) * np.sin(ph), np.cos(th)], -1).reshape(-1, 1, 3)
        vals = _lmarg_batch(dirs, a_q + a_k)
        assert vals.min() >= best - 1e-12


def test_bound_eq4_on_random_projectors():
    rng = np.random.default_rng(11)
    d = 8
    for _ in range(20):
        a_q = _rand_psd(rng, d, rank=rng.integers(1, d + 1))
        a_k = _rand_psd(rng, d, rank=rng.integers(1, d + 1))
        for r in range(0, d + 1):
            ms = _rand_projectors(rng, 50, d, r) if r else np.zeros((50, 0, d))
            m_star, _ = O.joint_basis(a_q[None], a_k[None], r) if r else (np.zeros((1, 0, d)), None)
            for m in list(ms) + [m_star[0]]:
                p = O.projector(m)
                c = np.eye(d) - p
                sel = O.l_sel(p, a_q, a_k)
                prod = np.trace(c @ a_q) * np.trace(c @ a_k)
                marg = O.l_marg(p, a_q, a_k)
                assert sel >= -1e-14
                assert sel <= prod + 1e-14
                assert prod <= 0.25 * marg * marg + 1e-14


def test_score_error_identity():
    # eq. (2): s - s_hat = q^T (I - P) k for any projector (checked against the two scores directly)
    rng = np.random.default_rng(12)
    d, r = 16, 5
    m = _rand_projectors(rng, 1, d, r)[0]
    p = O.projector(m)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    s = q @ k
    s_hat = (m @ q) @ (m @ k)
    assert abs((s - s_hat) - O.score_error(q, k, p)) <= 1e-12


def test_unit_trace_scale_invariance():
    rng = np.random.default_rng(13)
    d, r = 12, 4
    a_q = _rand_psd(rng, d)
    a_k = _rand_psd(rng, d)
    m1, _ = O.joint_basis(a_q[None], a_k[None], r)
    m2, _ = O.joint_basis(37.5 * a_q[None], 0.01 * a_k[None], r)
    assert np.max(np.abs(O.projector(m1[0]) - O.projector(m2[0]))) <= 1e-10


def test_eigh_against_independent_jacobi():
    rng = np.random.default_rng(14)
    for d in (5, 12, 24):
        a = _rand_psd(rng, d) + _rand_psd(rng, d)
        w_ref, u_ref = jacobi_eigh(a)
        m, w = O.joint_basis(_rand_psd(rng, d)[None] * 0 + a[None] / 2, a[None] / 2, d // 2)
        # joint_basis(a/2, a/2) normalises each to unit trace: eigenvalues are those of 2a/tr(a)
        scale = 2.0 / np.trace(a)
        assert np.allclose(np.sort(w[0]), w_ref * scale, atol=1e-12)
        p_ref = u_ref[:, ::-1][:, : d // 2] @ u_ref[:, ::-1][:, : d // 2].T
        assert np.max(np.abs(O.projector(m[0]) - p_ref)) <= 1e-9


def test_planted_mistakes_are_caught(tiny_calib):
    w, res = tiny_calib
    h = 0
    a_q = O.unit_trace(res["gram_q"][h])
    a_k = O.unit_trace(res["gram_k"][h])
    lam = res["eigvals"][h]
    # (1) taking the smallest eigenvectors breaks the Ky Fan value
    wv, u = np.linalg.eigh(a_q + a_k)
    m_bad = u[:, : w.rank].T
    assert abs(O.l_marg(O.projector(m_bad), a_q, a_k) - (2.0 - lam[: w.rank].sum())) > 1e-3
    # (2) skipping the unit-trace normalisation changes the subspace for unequal scales
    g_q, g_k = res["gram_q"][h], res["gram_k"][h]
    wv2, u2 = np.linalg.eigh(g_q + g_k)
    m_raw = u2[:, ::-1][:, : w.rank].T
    assert np.max(np.abs(O.projector(m_raw) - O.projector(res["M"][h]))) > 1e-3


def test_sign_rule_of_basis_rows():
    # each row keeps its direction and is signed so that its largest-magnitude entry is positive,
    # the lowest column winning a tie in magnitude
    rng = np.random.default_rng(15)
    m = rng.standard_normal((6, 9))
    s = O.sign_rows(m)
    for a, b in zip(m, s):
        assert np.allclose(np.abs(a), np.abs(b)) and (np.allclose(a, b) or np.allclose(a, -b))
        assert b[np.argmax(np.abs(b))] > 0
    tie = np.array([[-2.0, 2.0, 1.0], [2.0, -2.0, 0.5], [0.0, 0.0, 0.0]])
    out = O.sign_rows(tie)
    assert np.array_equal(out[0], [2.0, -2.0, -1.0])   # column 0 wins the tie, was negative
    assert np.array_equal(out[1], [2.0, -2.0, 0.5])    # column 0 wins, already positive
    assert np.array_equal(out[2], [0.0, 0.0, 0.0])     # a zero row stays as it is
    assert np.array_equal(O.sign_rows(out), out)        # idempotent
