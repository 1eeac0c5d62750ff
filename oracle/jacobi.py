"""Cyclic Jacobi eigensolver for small symmetric matrices (float64, pure NumPy).

Test infrastructure only. It is an independent second route to the eigendecomposition that the
joint basis needs (JSSA summary, eq. (5)), used to cross-check the LAPACK routine the oracle
calls; it is the textbook method (row-cyclic sweeps of 2x2 symmetric Schur rotations), not the
GPU's parallel ordering.
"""

from __future__ import annotations

import numpy as np


def jacobi_eigh(a: np.ndarray, tol: float = 1e-15, max_sweeps: int = 60) -> tuple:
    """Eigenvalues (ascending) and eigenvectors (columns) of symmetric ``a``."""
    a = np.array(a, dtype=np.float64, copy=True)
    n = a.shape[0]
    v = np.eye(n)
    norm = np.linalg.norm(a)
    for _ in range(max_sweeps):
        off = np.sqrt(max(0.0, np.sum(a * a) - np.sum(np.diag(a) ** 2)))
        if off <= tol * norm:
            break
        for p in range(n - 1):
            for q in range(p + 1, n):
                apq = a[p, q]
                if apq == 0.0:
                    continue
                tau = (a[q, q] - a[p, p]) / (2.0 * apq)
                t = (1.0 if tau >= 0 else -1.0) / (abs(tau) + np.sqrt(1.0 + tau * tau))
                c = 1.0 / np.sqrt(1.0 + t * t)
                s = t * c
                rot = np.eye(n)
                rot[p, p] = c
                rot[q, q] = c
                rot[p, q] = s
                rot[q, p] = -s
                a = rot.T @ a @ rot
                v = v @ rot
    w = np.diag(a).copy()
    order = np.argsort(w)
    return w[order], v[:, order]
