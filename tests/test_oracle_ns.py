"""Pins of the fp64 Newton-Schulz oracle against facts fixed by the mathematics.

None of these re-types the oracle's loop.  Each compares it with something
else: the scalar map on diagonal inputs, a closed form built from two
independent SVDs (LAPACK and a brute-force Jacobi), invariances, special cases,
the quintic's singular-value band around the polar factor ("nearest
semi-orthogonal matrix", "The NanoGPT speedrun", paragraph "Six records account
for most of the speedup"), and the FLOP figures that page prints.
"""
import json
import os

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from oracle import muon
from oracle.jacobi import jacobi_svd, polar_factor

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# The coefficient triple written out here, independently of the oracle's constant.
A_, B_, C_ = 3.4445, -4.7750, 2.0315


def p_iter(sigma, steps=5):
    """Scalar map sigma -> a s + b s^3 + c s^5, iterated ``steps`` times."""
    s = np.asarray(sigma, dtype=np.float64)
    for _ in range(steps):
        s = A_ * s + B_ * s ** 3 + C_ * s ** 5
    return s


def rect_diag(d, rows, cols):
    X = np.zeros((rows, cols))
    X[np.arange(len(d)), np.arange(len(d))] = d
    return X


def closed_form(X, svd, steps=5, eps=muon.NORM_EPS):
    """U diag(p^T(sigma / (||X||_F + eps))) V^T from the given SVD routine."""
    U, s, Vt = svd(X)
    nrm = np.sqrt(np.sum(np.asarray(X, float) ** 2)) + eps
    return (U * p_iter(s / nrm, steps)) @ Vt


def lapack_svd(X):
    return np.linalg.svd(X, full_matrices=False)


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def seeded_orthogonal(n, seed):
    q, r = np.linalg.qr(np.random.default_rng(seed).standard_normal((n, n)))
    return q * np.sign(np.diag(r))


def test_coefficients_are_the_specified_triple():
    assert muon.NS_COEFFS == (A_, B_, C_)
    assert muon.NS_STEPS == 5
    # p(1) = a + b + c: the map does not fix 1, it oscillates in a band.
    assert abs(sum(muon.NS_COEFFS) - 0.701) < 1e-12


@pytest.mark.parametrize("rows,cols", [(5, 5), (4, 9), (9, 4), (1, 7), (16, 16)])
def test_scalar_map_on_diagonal_inputs(rows, cols):
    rng = np.random.default_rng(rows * 100 + cols)
    k = min(rows, cols)
    d = rng.uniform(0.05, 2.0, size=k) * rng.choice([-1.0, 1.0], size=k)
    X = rect_diag(d, rows, cols)
    out = muon.newton_schulz(X, eps=0.0)
    expect = rect_diag(p_iter(d / np.linalg.norm(d)), rows, cols)
    assert np.max(np.abs(out - expect)) < 1e-13


def test_scalar_map_with_eps():
    d = np.array([3.0, -1.0, 0.5])
    out = muon.newton_schulz(np.diag(d))
    expect = np.diag(p_iter(d / (np.linalg.norm(d) + muon.NORM_EPS)))
    assert np.max(np.abs(out - expect)) < 1e-14


@pytest.mark.parametrize("shape", [(6, 11), (16, 16), (13, 4), (2, 3), (8, 40)])
def test_closed_form_lapack(shape):
    X = np.random.default_rng(sum(shape)).standard_normal(shape)
    assert rel(muon.newton_schulz(X), closed_form(X, lapack_svd)) < 1e-11


@pytest.mark.parametrize("shape", [(6, 11), (16, 16), (13, 4), (3, 3)])
def test_closed_form_jacobi(shape):
    X = np.random.default_rng(7 + sum(shape)).standard_normal(shape)
    assert rel(muon.newton_schulz(X), closed_form(X, jacobi_svd)) < 1e-11


@pytest.mark.parametrize("shape", [(5, 9), (9, 5), (16, 16), (1, 4)])
def test_jacobi_matches_lapack(shape):
    X = np.random.default_rng(3).standard_normal(shape)
    U, s, Vt = jacobi_svd(X)
    assert np.max(np.abs((U * s) @ Vt - X)) < 1e-12
    assert np.max(np.abs(s - np.linalg.svd(X, compute_uv=False))) < 1e-12
    assert np.max(np.abs(U.T @ U - np.eye(len(s)))) < 1e-12


@pytest.mark.parametrize("rows,cols", [(7, 12), (12, 7), (10, 10), (24, 64)])
def test_orthogonal_invariance(rows, cols):
    rng = np.random.default_rng(rows + 31 * cols)
    X = rng.standard_normal((rows, cols))
    Q, R = seeded_orthogonal(rows, 1), seeded_orthogonal(cols, 2)
    lhs = muon.newton_schulz(Q @ X @ R)
    rhs = Q @ muon.newton_schulz(X) @ R
    assert rel(lhs, rhs) < 1e-11


@pytest.mark.parametrize("rows,cols", [(5, 17), (17, 5), (30, 31)])
def test_transpose_symmetry(rows, cols):
    X = np.random.default_rng(rows * cols).standard_normal((rows, cols))
    assert rel(muon.newton_schulz(X.T), muon.newton_schulz(X).T) < 1e-13


@pytest.mark.parametrize("k", [1e-3, 0.5, 37.0, 2.0 ** 20])
def test_scale_invariance(k):
    X = np.random.default_rng(11).standard_normal((9, 14))
    assert rel(muon.newton_schulz(k * X, eps=0.0), muon.newton_schulz(X, eps=0.0)) < 1e-13
    # with the eps guard the difference is of order eps / ||X||
    assert rel(muon.newton_schulz(k * X), muon.newton_schulz(X)) < 1e-6 / min(k, 1.0)


def test_band_around_polar_factor():
    """Singular values with normalised sigma0 >= 2e-3 land in [0.6818, 1.2024]."""
    rng = np.random.default_rng(5)
    m, n = 12, 20
    U = seeded_orthogonal(m, 3)
    V = seeded_orthogonal(n, 4)[:m]
    sig0 = np.sort(10.0 ** rng.uniform(-2.5, 0, size=m))[::-1]
    X = (U * sig0) @ V
    sig_norm = sig0 / np.linalg.norm(sig0)
    out = muon.newton_schulz(X)
    s_out = np.linalg.svd(out, compute_uv=False)
    keep = sig_norm >= 2e-3
    assert keep.sum() >= 8
    s_keep = np.sort(s_out)[::-1][: keep.sum()]
    assert s_keep.min() >= 0.6818 - 1e-9 and s_keep.max() <= 1.2024 + 1e-9
    # distance to the polar factor on the kept directions
    P = polar_factor(X)
    Uk = U[:, keep]
    diff = Uk.T @ (out - P)
    assert np.linalg.norm(diff, 2) <= 0.318 + 1e-9
    # and the map's maximum on [0, 1]
    grid = np.linspace(0, 1, 200001)
    assert abs(p_iter(grid, 1).max() - 1.2024) < 1e-4


def test_zero_steps_is_normalisation():
    X = np.random.default_rng(9).standard_normal((6, 10))
    out = muon.newton_schulz(X, steps=0)
    assert rel(out, X / (np.linalg.norm(X) + muon.NORM_EPS)) < 1e-15
    assert abs(np.linalg.norm(muon.newton_schulz(X, steps=0, eps=0.0)) - 1.0) < 1e-14


@pytest.mark.parametrize("x", [3.0, -0.25, 1e-3])
def test_one_by_one(x):
    out = muon.newton_schulz(np.array([[x]]))
    assert out.shape == (1, 1)
    expect = p_iter(x / (abs(x) + muon.NORM_EPS))
    assert abs(out[0, 0] - expect) < 1e-12
    # iterating the map from 1 five times (eps = 0)
    assert abs(muon.newton_schulz(np.array([[x]]), eps=0.0)[0, 0] - np.sign(x) * p_iter(1.0)) < 1e-14


def test_zero_input_gives_zero():
    out = muon.newton_schulz(np.zeros((4, 7)))
    assert np.all(out == 0.0)


def test_flop_overhead_matches_page_figures():
    """T*m/B ~ 0.7 % ("The NanoGPT speedrun", record #3) from the FLOP formula.

    A square m x m hidden matrix costs 6*B*m^2 model FLOPs per step (forward
    and backward, 2 FLOPs per multiply-add); the iteration costs
    T*(4m^3 + 2m^3) = 6*T*m^3, so the ratio is exactly T*m/B.
    """
    with open(os.path.join(GOLDEN, "page_figures.json")) as f:
        fig = json.load(f)
    T, m, B = fig["T"], fig["m"], fig["B"]
    ratio = muon.ns_flops(m, m, T) / (6.0 * B * m * m)
    assert ratio == pytest.approx(T * m / B, rel=1e-15)
    assert abs(100 * ratio - fig["overhead_percent_printed"]) <= fig["overhead_percent_rounding"]
    # a 1:4 MLP matrix costs less than the bound ("at most")
    assert muon.ns_flops(m, 4 * m, T) / (6.0 * B * m * 4 * m) < T * m / B
    # GPT-2 small hidden set: 1630.7 nominal GFLOP per step
    from newton_schulz_12_b200.workloads import gpt2_small_shapes
    total = sum(muon.ns_flops(r, c, T) for r, c in gpt2_small_shapes())
    assert abs(total / 1e9 - 1630.7) < 0.05


@settings(max_examples=25, deadline=None)
@given(rows=st.integers(1, 12), cols=st.integers(1, 12), seed=st.integers(0, 2 ** 31 - 1),
       steps=st.integers(0, 6))
def test_closed_form_property(rows, cols, seed, steps):
    X = np.random.default_rng(seed).standard_normal((rows, cols))
    out = muon.newton_schulz(X, steps=steps)
    assert rel(out, closed_form(X, lapack_svd, steps)) < 1e-10
