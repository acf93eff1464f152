"""Pins of the refinements' oracles: cautious weight decay and NorMuon's
per-neuron rescale ("The NanoGPT speedrun", paragraph "Reading guide"; the
pages name both and give no formulas -- the readings are in oracle/muon.py).

Hand-worked cases (tests/golden/refinements_worked.json), closed-form
properties that follow from the readings (Frobenius norm kept, equal row RMS
when beta2 = 0, invariance under column rotations, row permutations, scale
homogeneity), the fp32 restatements against the fp64 definitions, and planted
mistakes that each break one of them.
"""
import json
import os

import numpy as np
import pytest

from oracle import muon
from oracle.fp32_ref import apply_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "refinements_worked.json")


def golden(kind):
    with open(GOLDEN) as f:
        return json.load(f)[kind]


# ------------------------------------------------------------ cautious decay
@pytest.mark.parametrize("case", golden("cautious"))
def test_cautious_worked_examples(case):
    W, O = np.array(case["W"]), np.array(case["O"])
    assert np.array_equal(muon.cautious_mask(W, O), np.array(case["mask"], float))
    got = muon.apply_update(W, O, case["lr"], case["wd"], case["scale"], cautious=True)
    assert np.array_equal(got, case["W_new"])
    plain = muon.apply_update(W, O, case["lr"], case["wd"], case["scale"])
    assert np.array_equal(plain, case["W_new_plain"])
    # the fp32 order gives the same dyadic values
    got32 = apply_f32(W, O, case["lr"], case["wd"], case["scale"], cautious=True)
    assert np.array_equal(got32, np.float32(case["W_new"]))


def test_cautious_special_cases():
    rng = np.random.default_rng(0)
    W = rng.standard_normal(2000)
    O = rng.standard_normal(2000)
    # no decay: cautious changes nothing
    assert np.array_equal(muon.apply_update(W, O, 0.1, 0.0, 1.0, cautious=True),
                          muon.apply_update(W, O, 0.1, 0.0, 1.0))
    # the update agrees in sign everywhere: plain decay
    Os = np.abs(O) * np.sign(W)
    assert np.array_equal(muon.apply_update(W, Os, 0.1, 0.3, 2.0, cautious=True),
                          muon.apply_update(W, Os, 0.1, 0.3, 2.0))
    # it disagrees everywhere: no decay at all
    assert np.array_equal(muon.apply_update(W, -Os, 0.1, 0.3, 2.0, cautious=True),
                          muon.apply_update(W, -Os, 0.1, 0.0, 2.0))


def test_cautious_f32_within_rounding():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal(5000) * 0.02).astype(np.float32)
    O = rng.standard_normal(5000).astype(np.float32)
    got = apply_f32(W, O, 0.05, 0.1, 2.0, cautious=True)
    lw = float(np.float32(np.float32(0.05) * np.float32(0.1)))   # the fp32 scalars, exactly
    ls = float(np.float32(np.float32(0.05) * np.float32(2.0)))
    ref = muon.apply_update(W, O, 1.0, lw, ls, cautious=True)    # W - lw mask W - ls O in fp64
    assert np.max(np.abs(got - ref)) <= 4 * np.spacing(np.float32(np.abs(ref).max()))
    mask32 = (W.astype(np.float64) * O > 0)
    assert np.array_equal(mask32, muon.cautious_mask(W, O) > 0)


@pytest.mark.parametrize("mutant", ["opposite_sign", "zero_decays"])
def test_cautious_planted_mistakes_fail(mutant):
    def bad_apply(W, O, lr, wd, scale):
        mask = (W * O < 0) if mutant == "opposite_sign" else (W * O >= 0)
        return W - lr * wd * W * mask - lr * scale * O
    case = golden("cautious")[0]
    W, O = np.array(case["W"]), np.array(case["O"])
    assert not np.array_equal(bad_apply(W, O, case["lr"], case["wd"], case["scale"]), case["W_new"])


def test_row_scale_in_fp32_order():
    rng = np.random.default_rng(2)
    W = rng.standard_normal((7, 9)).astype(np.float32)
    O = rng.standard_normal((7, 9)).astype(np.float32)
    assert np.array_equal(apply_f32(W, O, 0.05, 0.1, 1.0, row_scale=np.ones(7, np.float32)),
                          apply_f32(W, O, 0.05, 0.1, 1.0))
    f = np.float32(2.0 ** np.arange(-3, 4))
    assert np.array_equal(apply_f32(W, O, 0.05, 0.1, 1.0, row_scale=f),
                          apply_f32(W, O * f[:, None], 0.05, 0.1, 1.0))


# ---------------------------------------------------------------- NorMuon
@pytest.mark.parametrize("case", golden("normuon"))
def test_normuon_worked_examples(case):
    O, v = np.array(case["O"]), np.array(case["v"])
    got, v_new = muon.normuon_rescale(O, v, case["beta2"], case["eps"])
    assert np.array_equal(v_new, case["v_new"])
    np.testing.assert_allclose(got * got, case["O_new_squared"], rtol=1e-15, atol=0)
    assert np.all(np.sign(got) == np.sign(O))


def _rand(shape, seed):
    rng = np.random.default_rng(seed)
    O = rng.standard_normal(shape) * rng.uniform(0.1, 3.0, (shape[0], 1))  # uneven rows
    v = rng.uniform(0.0, 2.0, shape[0])
    return O, v


@pytest.mark.parametrize("shape", [(16, 40), (40, 16), (33, 33), (1, 9)])
def test_normuon_keeps_the_frobenius_norm(shape):
    O, v = _rand(shape, 3)
    for beta2 in (0.0, 0.5, 0.95, 1.0):
        got, _ = muon.normuon_rescale(O, v, beta2)
        assert np.isclose(np.linalg.norm(got), np.linalg.norm(O), rtol=1e-13)


def test_normuon_beta2_zero_equalises_row_rms():
    """With beta2 = 0 and no guard every row ends with the same RMS,
    ||O||_F / sqrt(rows cols): the per-neuron rescale's fixed point."""
    O, v = _rand((24, 56), 4)
    got, _ = muon.normuon_rescale(O, v, 0.0, eps=0.0)
    rms = np.sqrt(np.mean(got * got, axis=1))
    np.testing.assert_allclose(rms, np.linalg.norm(O) / np.sqrt(O.size), rtol=1e-13)
    got_eps, _ = muon.normuon_rescale(O, v, 0.0)  # the library's guard is negligible here
    np.testing.assert_allclose(got_eps, got, rtol=1e-8)


def test_normuon_column_rotation_invariance():
    """Row norms do not change under O -> O Q (Q orthogonal), so the rescale commutes with it."""
    O, v = _rand((12, 20), 5)
    Q, _ = np.linalg.qr(np.random.default_rng(6).standard_normal((20, 20)))
    a, va = muon.normuon_rescale(O @ Q, v, 0.9)
    b, vb = muon.normuon_rescale(O, v, 0.9)
    np.testing.assert_allclose(a, b @ Q, rtol=0, atol=1e-12)
    np.testing.assert_allclose(va, vb, rtol=1e-13)


def test_normuon_row_permutation_and_homogeneity():
    O, v = _rand((10, 14), 7)
    p = np.random.default_rng(8).permutation(10)
    a, va = muon.normuon_rescale(O[p], v[p], 0.8)
    b, vb = muon.normuon_rescale(O, v, 0.8)
    np.testing.assert_allclose(a, b[p], rtol=1e-14)
    np.testing.assert_allclose(va, vb[p], rtol=1e-14)
    # O -> k O with the state scaled by k^2: O' -> k O', v' -> k^2 v' (no guard)
    k = 3.0
    c, vc = muon.normuon_rescale(k * O, k * k * v, 0.8, eps=0.0)
    d, vd = muon.normuon_rescale(O, v, 0.8, eps=0.0)
    np.testing.assert_allclose(c, k * d, rtol=1e-13)
    np.testing.assert_allclose(vc, k * k * vd, rtol=1e-13)


def test_normuon_even_rows_change_nothing():
    """Rows of equal mean square and an even state: D is a multiple of I, O' = O."""
    Q, _ = np.linalg.qr(np.random.default_rng(9).standard_normal((32, 32)))
    O = Q[:8]  # orthonormal rows, mean square 1/32 each
    got, v_new = muon.normuon_rescale(O, np.full(8, 0.25), 0.9)
    np.testing.assert_allclose(got, O, rtol=0, atol=1e-14)
    np.testing.assert_allclose(v_new, 0.9 * 0.25 + 0.1 / 32, rtol=1e-14)


def test_normuon_zero_update():
    got, v_new = muon.normuon_rescale(np.zeros((4, 6)), np.ones(4), 0.5)
    assert np.all(got == 0) and np.array_equal(v_new, np.full(4, 0.5))


def test_step_ex_composes_the_refinements():
    rng = np.random.default_rng(10)
    W = rng.standard_normal((12, 20)) * 0.02
    g = rng.standard_normal((12, 20)) * 0.01
    buf = rng.standard_normal((12, 20)) * 0.01
    v = rng.uniform(0, 1e-3, 12)
    W2, nb, O2, v2 = muon.muon_step_ex(W, g, buf, lr=0.1, wd=0.2, cautious=True, neuron_state=v,
                                       beta2=0.9)
    nb_ref, u = muon.momentum(g, buf, 0.95, True)
    O = muon.newton_schulz(u)
    O_ref, v_ref = muon.normuon_rescale(O, v, 0.9)
    assert np.array_equal(nb, nb_ref) and np.array_equal(O2, O_ref) and np.array_equal(v2, v_ref)
    assert np.array_equal(W2, muon.apply_update(W, O_ref, 0.1, 0.2, 1.0, cautious=True))
    # without options it is muon_step
    a = muon.muon_step_ex(W, g, buf, lr=0.1, wd=0.2)
    b = muon.muon_step(W, g, buf, lr=0.1, wd=0.2)
    assert all(np.array_equal(x, y) for x, y in zip(a[:3], b)) and a[3] is None


def test_step_ex_schedule_is_the_ns_schedule():
    """A schedule only changes the orthogonalisation: the step with it is
    momentum -> newton_schulz(schedule) -> apply, and the default triple at
    every step is the plain step."""
    rng = np.random.default_rng(12)
    W = rng.standard_normal((10, 18)) * 0.02
    g = rng.standard_normal((10, 18)) * 0.01
    buf = rng.standard_normal((10, 18)) * 0.01
    sched = [(3.4445, -4.7750, 2.0315), (15 / 8, -10 / 8, 3 / 8), (1.5, -0.5, 0.0)]
    W2, nb, O2, _ = muon.muon_step_ex(W, g, buf, lr=0.1, wd=0.2, schedule=sched)
    _, u = muon.momentum(g, buf, 0.95, True)
    O = muon.newton_schulz(u, schedule=sched)
    assert np.array_equal(O2, O)
    assert np.array_equal(W2, muon.apply_update(W, O, 0.1, 0.2, muon.update_scale(10, 18)))
    a = muon.muon_step_ex(W, g, buf, lr=0.1, wd=0.2, schedule=[muon.NS_COEFFS] * muon.NS_STEPS)
    b = muon.muon_step_ex(W, g, buf, lr=0.1, wd=0.2)
    assert all(np.array_equal(x, y) for x, y in zip(a[:3], b[:3]))
    # and the order of the triples matters (the cubic first differs)
    c = muon.muon_step_ex(W, g, buf, lr=0.1, wd=0.2, schedule=sched[::-1])
    assert not np.allclose(c[2], O2, rtol=0, atol=1e-6)


def _mut_per_column(O, v, b2, eps):
    """statistics per column instead of per row (the wrong neuron axis)"""
    return muon.normuon_rescale(O.T, np.resize(v, O.shape[1]), b2, eps)[0].T


def _mut_no_renorm(O, v, b2, eps):
    """no renormalisation to ||O||_F"""
    return O / np.sqrt(b2 * v + (1 - b2) * np.mean(O * O, axis=1) + eps)[:, None]


def _mut_swapped_ema(O, v, b2, eps):
    """the moving average with its two weights swapped"""
    v_bad = (1 - b2) * v + b2 * np.mean(O * O, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):  # a mutant may divide by zero
        DO = O / np.sqrt(v_bad + eps)[:, None]
    return np.linalg.norm(O) / np.linalg.norm(DO) * DO


def _mut_no_sqrt(O, v, b2, eps):
    """dividing by the second moment instead of its root"""
    DO = O / (b2 * v + (1 - b2) * np.mean(O * O, axis=1) + eps)[:, None]
    return np.linalg.norm(O) / np.linalg.norm(DO) * DO


MUTANTS = {"per_column": _mut_per_column, "no_renorm": _mut_no_renorm,
           "swapped_ema": _mut_swapped_ema, "no_sqrt": _mut_no_sqrt}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_normuon_planted_mistakes_fail(name):
    bad = MUTANTS[name]
    caught = False
    for case in golden("normuon"):
        O, v = np.array(case["O"]), np.array(case["v"])
        got = bad(O, v, case["beta2"], case["eps"])
        if got.shape != O.shape or not np.allclose(got * got, case["O_new_squared"], rtol=1e-12):
            caught = True
    O, v = _rand((12, 30), 11)
    got = bad(O, v, 0.0, 0.0)
    if got.shape != O.shape or not np.isclose(np.linalg.norm(got), np.linalg.norm(O), rtol=1e-12):
        caught = True
    rms = np.sqrt(np.mean(got * got, axis=1))
    if not np.allclose(rms, np.linalg.norm(O) / np.sqrt(O.size), rtol=1e-10):
        caught = True
    assert caught, name
