"""Pins of the oracle's per-step coefficient schedule (Polar Express form).

"The NanoGPT speedrun", paragraph "Reading guide", names Polar Express
polynomials among the later refinements of the same update: the iteration
keeps its form X <- aX + (bA + cA^2)X but each step has its own (a, b, c).
The pages print no coefficients, so these pins use triples chosen here and
check the oracle against mathematics that does not share its loop: on a
(rectangular) diagonal input each singular value follows the composition of
the per-step scalar maps, applied in order; orthogonal transforms commute
with the iteration; a constant schedule is the fixed-triple iteration.
"""
import numpy as np
import pytest

from oracle import muon

# Triples written out here: the speedrun quintic, the classic cubic
# 1.5 x - 0.5 x^3, and the quintic with p(1) = 1, p'(1) = p''(1) = 0.
QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)
FLAT = (15 / 8, -10 / 8, 3 / 8)
SCHEDULE = [QUINTIC, QUINTIC, CUBIC, FLAT, CUBIC]


def scalar_chain(sigma, schedule):
    """sigma -> a_t s + b_t s^3 + c_t s^5 for t = 1, 2, ... in plain floats."""
    out = []
    for s in sigma:
        s = float(s)
        for a, b, c in schedule:
            s = a * s + b * s ** 3 + c * s ** 5
        out.append(s)
    return np.array(out)


def rect_diag(d, rows, cols):
    X = np.zeros((rows, cols))
    X[np.arange(len(d)), np.arange(len(d))] = d
    return X


@pytest.mark.parametrize("rows,cols", [(4, 4), (3, 7), (7, 3)])
def test_diagonal_follows_the_composed_scalar_maps(rows, cols):
    d = np.array([0.9, 0.5, 0.1][: min(rows, cols)] + [0.02] * (min(rows, cols) - 3))
    X = rect_diag(d, rows, cols)
    got = np.diag(muon.newton_schulz(X, schedule=SCHEDULE))
    want = scalar_chain(d / (np.linalg.norm(d) + muon.NORM_EPS), SCHEDULE)
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-15)


def test_order_of_the_schedule_matters():
    """The per-step maps do not commute: applying the schedule reversed is a
    different function, and the diagonal pin tells the two apart."""
    d = np.array([0.9, 0.3, 0.05])
    X = np.diag(d)
    fwd = np.diag(muon.newton_schulz(X, schedule=SCHEDULE))
    rev = np.diag(muon.newton_schulz(X, schedule=SCHEDULE[::-1]))
    want = scalar_chain(d / (np.linalg.norm(d) + muon.NORM_EPS), SCHEDULE)
    np.testing.assert_allclose(fwd, want, rtol=1e-13)
    assert np.max(np.abs(rev - want)) > 1e-3


def test_constant_schedule_is_the_fixed_triple_iteration():
    G = np.random.default_rng(1).standard_normal((24, 40))
    np.testing.assert_array_equal(muon.newton_schulz(G, schedule=[QUINTIC] * 5),
                                  muon.newton_schulz(G, steps=5, coeffs=QUINTIC))


def test_empty_schedule_is_the_normalised_input():
    G = np.random.default_rng(2).standard_normal((9, 5))
    np.testing.assert_allclose(muon.newton_schulz(G, schedule=[]),
                               G / (np.linalg.norm(G) + muon.NORM_EPS), rtol=1e-15)


def test_orthogonal_invariance_with_a_schedule():
    rng = np.random.default_rng(3)
    G = rng.standard_normal((12, 20))
    U, _ = np.linalg.qr(rng.standard_normal((12, 12)))
    V, _ = np.linalg.qr(rng.standard_normal((20, 20)))
    lhs = muon.newton_schulz(U @ G @ V, schedule=SCHEDULE)
    rhs = U @ muon.newton_schulz(G, schedule=SCHEDULE) @ V
    np.testing.assert_allclose(lhs, rhs, atol=1e-12)


def test_singular_values_follow_the_chain_on_a_dense_input():
    """Dense input: NS(X) = U diag(p_T o ... o p_1 (s / ||X||)) V^T."""
    rng = np.random.default_rng(4)
    G = rng.standard_normal((16, 30))
    U, s, Vt = np.linalg.svd(G, full_matrices=False)
    want = U @ np.diag(scalar_chain(s / (np.linalg.norm(G) + muon.NORM_EPS), SCHEDULE)) @ Vt
    np.testing.assert_allclose(muon.newton_schulz(G, schedule=SCHEDULE), want, atol=1e-12)
