"""Pins of the synthetic selection-quality report (``oracle/selection_quality.py``; JSSA summary,
Theoretical Foundation, eqs. (3)-(5), and the basis comparison of its ablations).

* With the full rank r = d every basis (joint, keys only, queries only) is an orthonormal basis of
  the whole space, so M^T M = I and the float64 projected score equals the exact group-mean score:
  the report's float64 row must give recall 1 and keep all of the exact top-B's attention mass.
* The attention mass it averages is a distribution over positions (each head's softmax sums to
  one), and the mass of the exact top-B is the largest any B positions carry for the head mean.
* A planted mistake, a rank-deficient "full" basis, loses recall.
"""

import numpy as np

from oracle import jssa as O
from oracle import selection_quality as SQ


def test_full_rank_float64_scores_recall_everything():
    d = 64
    out = SQ.run(seq_len=2048, budget=64, n_queries=2, ranks=(d,), seed=1711, h_kv=2, group=2,
                 d=d, n_calib=2048)
    row = out["rows"][("joint, float64 scores", d)]
    assert len(row["recall"]) == 2 * 2
    np.testing.assert_allclose(row["recall"], 1.0)
    np.testing.assert_allclose(row["mass"], 1.0, rtol=1e-12)
    # every full-rank basis is orthonormal and complete
    rng = np.random.default_rng(3)
    g = rng.standard_normal((2, d, d))
    g_q = np.einsum("hij,hkj->hik", g, g)
    g_k = np.einsum("hij,hkj->hik", g[::-1], g[::-1])
    for name, m in SQ.bases(g_q, g_k, d).items():
        np.testing.assert_allclose(np.einsum("hri,hrj->hij", m, m),
                                   np.broadcast_to(np.eye(d), (2, d, d)), atol=1e-10, err_msg=name)


def test_attention_mass_is_a_distribution_and_top_b_maximises_it():
    rng = np.random.default_rng(5)
    k = rng.standard_normal((500, 16))
    qg = rng.standard_normal((4, 16))
    mass = SQ.attention_mass(k, qg, 0.25)
    assert np.all(mass > 0)
    np.testing.assert_allclose(mass.sum(), 1.0, rtol=1e-12)
    # per head: the plain softmax of that head, averaged
    z = 0.25 * (k @ qg.T)
    p = np.exp(z - z.max(axis=0)) / np.exp(z - z.max(axis=0)).sum(axis=0)
    np.testing.assert_allclose(mass, p.mean(axis=1), rtol=1e-12)
    # with one head, the top-B of that head's score carries the most mass of any B positions
    m1 = SQ.attention_mass(k, qg[:1], 0.25)
    top = O.select_top_b(k @ qg[0], 50)
    assert m1[top].sum() >= np.sort(m1)[::-1][:50].sum() - 1e-12


def test_planted_rank_deficient_basis_loses_recall():
    # a "full" basis with one row repeated spans only d - 1 dimensions: its float64 scores are no
    # longer the exact ones, and the recall drops below 1
    d, budget = 32, 32
    rng = np.random.default_rng(7)
    k = rng.standard_normal((4096, d))
    qbar = rng.standard_normal(d)
    exact = O.select_top_b(k @ qbar, budget)
    q_, _ = np.linalg.qr(rng.standard_normal((d, d)))
    m = q_.T.copy()
    m[-1] = m[0]
    sel = O.select_top_b((k @ m.T) @ (m @ qbar), budget)
    assert np.intersect1d(sel, exact).size < budget
    sel_full = O.select_top_b((k @ q_) @ (q_.T @ qbar), budget)
    assert np.intersect1d(sel_full, exact).size == budget
