"""Planted mistakes: each plausible slip in the oracle must fail at least one pin.

The mutants are copies of the oracle's Newton-Schulz with one mistake planted
(on the CPU).  The pin battery below is the same set of facts the real oracle
passes in test_oracle_ns.py: scalar map on diagonals, the SVD closed form,
orthogonal invariance and transpose symmetry.
"""
import warnings

import numpy as np
import pytest

from oracle import muon

from test_oracle_ns import closed_form, lapack_svd, p_iter, rect_diag, rel, seeded_orthogonal


def make_ns(mistake=None):
    a, b, c = muon.NS_COEFFS
    if mistake == "sign_c":
        c = -c
    if mistake == "swap_ab":
        a, b = b, a

    def ns(G, steps=5, eps=muon.NORM_EPS):
        X = np.asarray(G, dtype=np.float64)
        tr = X.shape[0] > X.shape[1]
        if tr and mistake != "no_transpose":
            X = X.T
        if mistake != "no_normalise":
            X = X / (np.sqrt(np.sum(X * X)) + eps)
        for _ in range(steps if mistake != "one_step_short" else steps - 1):
            A = X @ X.T if mistake != "gram_swapped" else X.T @ X
            if mistake == "drop_A_term":
                B = c * (A @ A)
            else:
                B = b * A + c * (A @ A)
            if mistake == "drop_aX":
                X = B @ X
            elif mistake == "right_multiply":
                X = a * X + X @ B if B.shape[0] == X.shape[1] else a * X + B @ X
            else:
                X = a * X + B @ X
        if tr and mistake not in ("no_transpose", "forget_untranspose"):
            X = X.T
        return X

    return ns


def pins_hold(ns):
    """True when every pin holds; a NaN or overflow counts as a failure."""
    try:
        # scalar map on rectangular diagonals
        for rows, cols in ((4, 9), (9, 4), (5, 5)):
            d = np.linspace(0.3, 1.7, min(rows, cols)) * np.array([1, -1] * 5)[: min(rows, cols)]
            out = ns(rect_diag(d, rows, cols), eps=0.0)
            if out.shape != (rows, cols):
                return False
            if not np.max(np.abs(out - rect_diag(p_iter(d / np.linalg.norm(d)), rows, cols))) <= 1e-12:
                return False
        # closed form, square and rectangular
        for shape in ((6, 6), (5, 11), (11, 5)):
            X = np.random.default_rng(sum(shape)).standard_normal(shape)
            out = ns(X)
            if out.shape != shape or not rel(out, closed_form(X, lapack_svd)) <= 1e-10:
                return False
        # orthogonal invariance on a square input
        X = np.random.default_rng(1).standard_normal((7, 7))
        Q, R = seeded_orthogonal(7, 1), seeded_orthogonal(7, 2)
        if not rel(ns(Q @ X @ R), Q @ ns(X) @ R) <= 1e-10:
            return False
        # transpose symmetry
        X = np.random.default_rng(2).standard_normal((5, 8))
        if not rel(ns(X.T), ns(X).T) <= 1e-12:
            return False
    except ValueError:  # shape mismatch inside the mutant
        return False
    return True


def test_real_oracle_passes_the_battery():
    assert pins_hold(muon.newton_schulz)
    assert pins_hold(make_ns(None))


# Not a mistake: skipping the transpose of a tall input gives the same function
# (aX + b(XX^T)X + c(XX^T)^2 X = aX + bX(X^TX) + cX(X^TX)^2), only dearer.
@pytest.mark.parametrize("mistake", ["sign_c", "swap_ab", "no_normalise",
                                     "one_step_short", "gram_swapped", "drop_A_term", "drop_aX",
                                     "right_multiply", "forget_untranspose"])
def test_planted_mistake_is_caught(mistake):
    with warnings.catch_warnings():
        warnings.simplefilter("ignore", RuntimeWarning)
        assert not pins_hold(make_ns(mistake))
