"""Pins of the oracle's second moments and calibration against the selection objective itself.

The pages define the joint basis through the token-score preservation error (JSSA summary,
"Theoretical Foundation", eqs. (2)-(3)): for a projector ``P`` the score error of a group-mean
query ``qbar`` and a key ``k`` is ``qbar^T (I - P) k``, and its expected square over queries and
keys drawn independently is ``tr((I - P) A_Q (I - P) A_K)`` with ``A_Q``, ``A_K`` the second
moments of the group-mean queries and of the keys. Over a finite calibration set the expectation
is a plain double sum over (query sample, key sample) pairs, so

    sum_{n, m} (qbar_n^T (I - P) k_m)^2 = tr((I - P) G_Q (I - P) G_K)

holds exactly for the uncentred sums ``G_Q = sum_n qbar_n qbar_n^T`` and ``G_K = sum_m k_m k_m^T``
and for every projector. Several random projectors determine a symmetric ``G_Q`` (and ``G_K``)
completely, so the identity pins ``second_moments`` and the Grams that ``calibrate`` returns: a
per-head moment ``(1/G) sum_g q_g q_g^T`` in place of ``qbar qbar^T``, a centred moment, or a
transposed or mis-indexed head would break it. The left side is computed pair by pair with the
oracle's score error (eq. (2)), which ``test_score_error_identity`` pins against the two scores.

With ``P = 0`` the identity reads ``sum_{n,m} (qbar_n . k_m)^2 = tr(G_Q G_K)``, and the unit-trace
form divides both sides by ``tr G_Q tr G_K`` (eq. (3) with ``A = G / tr G``).
"""

import numpy as np
import pytest

from oracle import jssa as O


def _rand_projector(rng, d, r):
    if r == 0:
        return np.zeros((d, d))
    q, _ = np.linalg.qr(rng.standard_normal((d, r)))
    return q @ q.T


def _samples(rng, n, h_q, h_kv, d, mean_shift=0.0):
    q = rng.standard_normal((n, h_q, d)) + mean_shift
    k = rng.standard_normal((n, h_kv, d)) * np.linspace(0.5, 2.0, d) + mean_shift
    return q, k


def _pair_sum(qbar_h, k_h, p):
    """sum over every (query sample, key sample) pair of the squared score error, eq. (2)."""
    total = 0.0
    for qn in qbar_h:
        for km in k_h:
            total += O.score_error(qn, km, p) ** 2
    return total


def _worst_mismatch(q, k, gram_q, gram_k, rng, projectors=6):
    """Largest relative gap between the pair sum and the trace form over random projectors of
    every rank, for each KV head."""
    h_kv, d = k.shape[1], k.shape[2]
    qbar = O.group_mean_query(q, h_kv)
    worst = 0.0
    for h in range(h_kv):
        for i in range(projectors):
            p = _rand_projector(rng, d, i % (d + 1))
            lhs = _pair_sum(qbar[:, h], k[:, h], p)
            rhs = O.l_sel(p, gram_q[h], gram_k[h])
            worst = max(worst, abs(lhs - rhs) / max(abs(lhs), 1e-300))
    return worst


@pytest.mark.parametrize("h_q,h_kv,d", [(6, 2, 5), (8, 2, 7), (4, 4, 6)])
def test_pair_sum_identity_pins_second_moments(h_q, h_kv, d):
    rng = np.random.default_rng(300 + h_q + d)
    q, k = _samples(rng, 23, h_q, h_kv, d, mean_shift=0.3)
    qbar = O.group_mean_query(q, h_kv)
    g_q, g_k = O.second_moments(qbar, k)
    assert _worst_mismatch(q, k, g_q, g_k, rng) <= 1e-11


def test_pair_sum_identity_pins_calibrate():
    rng = np.random.default_rng(310)
    h_q, h_kv, d, r = 8, 2, 6, 3
    q, k = _samples(rng, 31, h_q, h_kv, d, mean_shift=0.5)
    res = O.calibrate(q, k, r)
    assert _worst_mismatch(q, k, res["gram_q"], res["gram_k"], rng) <= 1e-11
    qbar = O.group_mean_query(q, h_kv)
    for h in range(h_kv):
        # P = 0: the plain double sum of squared scores
        direct = sum(float(qn @ km) ** 2 for qn in qbar[:, h] for km in k[:, h])
        assert abs(direct - np.trace(res["gram_q"][h] @ res["gram_k"][h])) <= 1e-11 * direct
        # the unit-trace form of eq. (3) at the calibrated projector
        p = O.projector(res["M"][h])
        a_q, a_k = O.unit_trace(res["gram_q"][h]), O.unit_trace(res["gram_k"][h])
        tr_q = sum(float(qn @ qn) for qn in qbar[:, h])
        tr_k = sum(float(km @ km) for km in k[:, h])
        lhs = _pair_sum(qbar[:, h], k[:, h], p) / (tr_q * tr_k)
        assert abs(lhs - O.l_sel(p, a_q, a_k)) <= 1e-11 * max(lhs, 1e-300)


def test_group_mean_query_head_mapping():
    # query head i belongs to KV head i // G: a query whose only non-zero head is i moves only
    # the group mean of KV head i // G, by 1/G of that head
    h_q, h_kv, d = 8, 2, 3
    g = h_q // h_kv
    for i in range(h_q):
        q = np.zeros((1, h_q, d))
        q[0, i] = [1.0, 2.0, 3.0]
        qbar = O.group_mean_query(q, h_kv)
        for h in range(h_kv):
            want = q[0, i] / g if h == i // g else np.zeros(d)
            assert np.array_equal(qbar[0, h], want)


def _per_head_moment_calibrate(q, k, r):
    """A plausible mistake: the average of the per-head moments (1/G) sum_g q_g q_g^T in place
    of the moment of the group mean."""
    n, h_q, d = q.shape
    h_kv = k.shape[1]
    g = h_q // h_kv
    g_q = np.einsum("nhgi,nhgj->hij", q.reshape(n, h_kv, g, d), q.reshape(n, h_kv, g, d)) / g
    g_k = np.einsum("nhi,nhj->hij", k, k)
    return g_q, g_k


def _centred_second_moments(qbar, k):
    """A plausible mistake: covariances (centred) instead of uncentred second moments."""
    qc = qbar - qbar.mean(axis=0, keepdims=True)
    kc = k - k.mean(axis=0, keepdims=True)
    return np.einsum("nhi,nhj->hij", qc, qc), np.einsum("nhi,nhj->hij", kc, kc)


def _misindexed_second_moments(qbar, k):
    """A plausible mistake: the query moment of KV head h taken from another head's group.
    (Swapping the query and key moments is not a mistake: the objective is symmetric in them.)"""
    return (np.einsum("nhi,nhj->hij", qbar[:, ::-1], qbar[:, ::-1]),
            np.einsum("nhi,nhj->hij", k, k))


def test_planted_moment_mistakes_are_caught(monkeypatch):
    rng = np.random.default_rng(320)
    h_q, h_kv, d, r = 8, 2, 6, 3
    q, k = _samples(rng, 29, h_q, h_kv, d, mean_shift=0.5)
    # the per-head moment
    g_q, g_k = _per_head_moment_calibrate(q, k, r)
    assert _worst_mismatch(q, k, g_q, g_k, rng) > 1e-3
    # a centred or mis-indexed second_moments, planted in the oracle and reached through calibrate
    for planted in (_centred_second_moments, _misindexed_second_moments):
        monkeypatch.setattr(O, "second_moments", planted)
        res = O.calibrate(q, k, r)
        assert _worst_mismatch(q, k, res["gram_q"], res["gram_k"], rng) > 1e-3
        monkeypatch.undo()
    # and the unplanted oracle passes on the same data
    res = O.calibrate(q, k, r)
    assert _worst_mismatch(q, k, res["gram_q"], res["gram_k"], rng) <= 1e-11
