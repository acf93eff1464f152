"""One-sided (Hestenes) Jacobi SVD for tiny matrices (test infrastructure only).

A brute-force route to the polar factor U V^T -- the "nearest semi-orthogonal
matrix" of "The NanoGPT speedrun", paragraph "Six records account for most of
the speedup" -- that shares nothing with LAPACK, so the oracle can be checked
against two independent SVDs.

Method (Hestenes 1958): rotate pairs of columns of a working copy of X until
all columns are mutually orthogonal; the column norms are then the singular
values, the normalised columns the left singular vectors, and the accumulated
rotations the right singular vectors.
"""
from __future__ import annotations

import numpy as np


def jacobi_svd(X, tol=1e-15, max_sweeps=100):
    """Thin SVD of a small fp64 matrix: returns (U, s, Vt) with X = U diag(s) Vt.

    Works on rows >= cols; a wide input is handled through its transpose.
    Singular values are returned in descending order.
    """
    X = np.array(X, dtype=np.float64)
    if X.shape[0] < X.shape[1]:
        U, s, Vt = jacobi_svd(X.T, tol, max_sweeps)
        return Vt.T, s, U.T
    _, n = X.shape
    Wk = X.copy()
    V = np.eye(n)
    for _ in range(max_sweeps):
        rotated = False
        for p in range(n - 1):
            for q in range(p + 1, n):
                alpha = float(Wk[:, p] @ Wk[:, p])
                beta = float(Wk[:, q] @ Wk[:, q])
                gamma = float(Wk[:, p] @ Wk[:, q])
                if abs(gamma) <= tol * np.sqrt(alpha * beta) or gamma == 0.0:
                    continue
                rotated = True
                zeta = (beta - alpha) / (2.0 * gamma)
                t = np.sign(zeta) / (abs(zeta) + np.sqrt(1.0 + zeta * zeta)) if zeta != 0 else 1.0
                cs = 1.0 / np.sqrt(1.0 + t * t)
                sn = cs * t
                wp, wq = Wk[:, p].copy(), Wk[:, q].copy()
                Wk[:, p] = cs * wp - sn * wq
                Wk[:, q] = sn * wp + cs * wq
                vp, vq = V[:, p].copy(), V[:, q].copy()
                V[:, p] = cs * vp - sn * vq
                V[:, q] = sn * vp + cs * vq
        if not rotated:
            break
    s = np.sqrt(np.sum(Wk * Wk, axis=0))
    order = np.argsort(-s)
    s = s[order]
    Wk = Wk[:, order]
    V = V[:, order]
    U = np.zeros_like(Wk)
    nz = s > 0
    U[:, nz] = Wk[:, nz] / s[nz]
    return U, s, V.T


def polar_factor(X):
    """U V^T from the Jacobi SVD (full column/row rank assumed)."""
    U, _, Vt = jacobi_svd(X)
    return U @ Vt
