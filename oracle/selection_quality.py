"""Synthetic selection-quality report: how close the top-B positions picked from projected FP8
scores come to the exact top-B of the full-dimension group-mean scores, and how much attention
mass they keep, for the joint basis and for key-only and query-only bases of the same rank.

A data-free analogue of the pages' basis comparison (JSSA summary, Theoretical Foundation and
eqs. (3)-(5): the joint basis minimises the marginal bound on the score error for queries and
keys together; JSSA README, "Highlights"). Analysis on the float64 oracle only (test
infrastructure), on the seeded low-rank generator of the 128K Llama-like layer (d 128, 8 KV
heads, 4 query heads each). Run from the repository root:

    python -m oracle.selection_quality [--seq-len 16384] [--budget 256] [--queries 4]
"""

from __future__ import annotations

import argparse

import numpy as np

from . import jssa as O


def top_eig_rows(a: np.ndarray, r: int) -> np.ndarray:
    """Rows = eigenvectors of the r largest eigenvalues of each symmetric ``a[h]`` (signed as the
    joint basis), i.e. the rank-r PCA basis of one unit-trace second moment."""
    w, u = np.linalg.eigh(a)
    m = np.swapaxes(u[..., ::-1][..., :r], -1, -2)
    return O.sign_rows(m)


def bases(g_q: np.ndarray, g_k: np.ndarray, r: int) -> dict:
    return {
        "joint (JSSA)": O.joint_basis(g_q, g_k, r)[0],
        "keys only": top_eig_rows(O.unit_trace(g_k), r),
        "queries only": top_eig_rows(O.unit_trace(g_q), r),
    }


def attention_mass(k: np.ndarray, qg: np.ndarray, scale: float) -> np.ndarray:
    """Per position, the softmax weight averaged over the group's query heads."""
    z = scale * (k @ qg.T)                   # [L, G]
    z = z - z.max(axis=0, keepdims=True)
    a = np.exp(z)
    a = a / a.sum(axis=0, keepdims=True)
    return a.mean(axis=1)


def run(seq_len: int, budget: int, n_queries: int, ranks=(4, 8, 16, 32), seed: int = 1002,
        h_kv: int = 8, group: int = 4, d: int = 128, n_calib: int = 32768) -> dict:
    from synth import layer_factors, sample_calibration, sample_decode_queries

    f = layer_factors(seed, 0, h_kv, d)
    qc, kc = sample_calibration(f, n_calib, group, seed)
    qbar_c = O.group_mean_query(qc.double().numpy(), h_kv)
    g_q, g_k = O.second_moments(qbar_c, kc.double().numpy())
    # cached keys: a fresh stream of the same layer's key distribution
    _, keys = sample_calibration(f, seq_len, group, seed, layer=7)
    keys = keys.double().numpy()             # [L, h_kv, d]
    scale = 1.0 / np.sqrt(d)
    res = {}
    for r in ranks:
        bs = bases(g_q, g_k, r)
        for name in bs:
            res[(name, r)] = {"recall": [], "mass": []}
        if r == max(ranks):
            res[("joint, float64 scores", r)] = {"recall": [], "mass": []}
    exact_mass = []
    for i in range(n_queries):
        q = sample_decode_queries(f, 1, group, seed, step=i)[0].double().numpy()  # [h_q, d]
        for h in range(h_kv):
            k = keys[:, h]
            qg = q[h * group:(h + 1) * group]
            qbar = qg.mean(axis=0)
            s_exact = k @ qbar
            s_star = O.select_top_b(s_exact, budget)
            mass = attention_mass(k, qg, scale)
            m_star = mass[s_star].sum()
            exact_mass.append(m_star)
            for r in ranks:
                for name, m in bases(g_q, g_k, r).items():
                    s = O.scores(O.store_codes(k, m[h]), O.projected_query(qbar, m[h]))
                    sel = O.select_top_b(s, budget)
                    res[(name, r)]["recall"].append(np.intersect1d(sel, s_star).size / budget)
                    res[(name, r)]["mass"].append(mass[sel].sum() / m_star)
                if r == max(ranks):
                    m = O.joint_basis(g_q, g_k, r)[0][h]
                    sel = O.select_top_b((k @ m.T) @ (m @ qbar), budget)
                    res[("joint, float64 scores", r)]["recall"].append(
                        np.intersect1d(sel, s_star).size / budget)
                    res[("joint, float64 scores", r)]["mass"].append(mass[sel].sum() / m_star)
    return {"rows": res, "exact_mass": float(np.mean(exact_mass))}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--seq-len", type=int, default=16384)
    ap.add_argument("--budget", type=int, default=256)
    ap.add_argument("--queries", type=int, default=4)
    a = ap.parse_args()
    out = run(a.seq_len, a.budget, a.queries)
    n = a.queries * 8
    print(f"L {a.seq_len}, B {a.budget}, {n} (decode query, KV head) pairs; attention mass of the "
          f"exact group-mean top-B: {out['exact_mass']:.4f} (mean over pairs)\n")
    print("| basis | r | recall of the exact top-B | attention mass kept (vs exact top-B) |")
    print("|---|---:|---:|---:|")
    for (name, r), v in sorted(out["rows"].items(), key=lambda x: (x[0][1], x[0][0])):
        print(f"| {name} | {r} | {np.mean(v['recall']):.3f} | {np.mean(v['mass']):.3f} |")


if __name__ == "__main__":
    main()
