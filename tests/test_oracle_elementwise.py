"""Pins of the momentum / scale / apply oracles (fp64 definition and fp32 order).

Hand-worked dyadic examples (tests/golden/momentum_worked.json), special cases
that collapse the formulas, agreement of the fp32 restatement with the fp64
definition within fp32 rounding, and the bf16 rounding helper against torch's
own bf16 cast.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import muon
from oracle.fp32_ref import apply_f32, bf16_round, momentum_f32, update_scale_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_cases():
    with open(os.path.join(GOLDEN, "momentum_worked.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", load_cases())
def test_momentum_worked_examples(case):
    g, buf = np.array(case["g"]), np.array(case["buf"])
    nb, u = muon.momentum(g, buf, case["beta"], case["nesterov"])
    assert np.array_equal(nb, case["buf_new"]) and np.array_equal(u, case["u"])
    nb32, u32 = momentum_f32(g, buf, case["beta"], case["nesterov"])
    assert np.array_equal(nb32, np.float32(case["buf_new"]))
    assert np.array_equal(u32, np.float32(case["u"]))


def test_momentum_special_cases():
    rng = np.random.default_rng(0)
    g, buf = rng.standard_normal(100), rng.standard_normal(100)
    nb, u = muon.momentum(g, buf, 1.0, True)
    assert np.array_equal(nb, buf) and np.array_equal(u, buf)
    nb, u = muon.momentum(g, buf, 0.0, False)
    assert np.array_equal(nb, g) and np.array_equal(u, g)
    # with zero initial buffer the classic Nesterov form U = g + beta*(beta*0 + g)
    # is (1+beta) g, the lerp form gives (1-beta)(1+beta) g: same direction.
    nb, u = muon.momentum(g, np.zeros_like(g), 0.95, True)
    assert np.allclose(u, (1 - 0.95) * (1 + 0.95) * g, rtol=1e-14, atol=0)


def test_momentum_f32_within_rounding_of_fp64():
    rng = np.random.default_rng(1)
    g = bf16_round(rng.standard_normal(4096).astype(np.float32) * 0.01)
    buf = rng.standard_normal(4096).astype(np.float32) * 0.01
    nb32, u32 = momentum_f32(g, buf, 0.95, True)
    b = np.float64(np.float32(0.95))
    nb64, u64 = muon.momentum(g.astype(np.float64), buf.astype(np.float64), b, True)
    # each fp32 rounding contributes at most 2^-24 of the magnitude it rounds
    u = 2.0 ** -24
    t1, t2 = np.abs(b * buf), np.abs((1 - b) * g)
    assert np.all(np.abs(nb32 - nb64) <= u * (t1 + t2 + np.abs(nb64)) * 1.01)
    t3 = np.abs(b * nb64)
    bound = u * (t2 + t3 + np.abs(u64)) + b * u * (t1 + t2 + np.abs(nb64))
    assert np.all(np.abs(u32 - u64) <= bound * 1.01)


def test_scale_rule():
    assert muon.update_scale(3072, 768) == 2.0
    assert muon.update_scale(768, 3072) == 1.0
    assert muon.update_scale(768, 768) == 1.0
    assert update_scale_f32(3072, 768) == np.float32(2.0)
    assert update_scale_f32(4096, 1024) == np.float32(2.0)
    assert update_scale_f32(768, 3072) == np.float32(1.0)
    assert update_scale_f32(300, 100) == np.float32(np.sqrt(np.float32(3.0)))


def test_apply_special_cases_and_rounding():
    rng = np.random.default_rng(2)
    W = rng.standard_normal(1000).astype(np.float32)
    O = rng.standard_normal(1000).astype(np.float32)
    assert np.array_equal(apply_f32(W, O, 0.0, 0.1, 1.0), W)
    assert np.array_equal(apply_f32(W, O, 0.05, 0.0, 1.0), W - np.float32(0.05) * O)
    # decoupled decay only: W (1 - lr wd)
    np.testing.assert_allclose(apply_f32(W, np.zeros_like(O), 0.5, 0.5, 1.0), 0.75 * W, rtol=1e-7)
    ref = muon.apply_update(W, O, 0.05, 0.01, 2.0)
    got = apply_f32(W, O, 0.05, 0.01, 2.0)
    assert np.max(np.abs(got - ref)) <= 4 * np.spacing(np.float32(np.abs(ref).max()))


def test_bf16_round_matches_torch_cast():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 10.0 ** rng.integers(-30, 30, 10000),
                        np.float32([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 3.0e38, -1e-40, np.inf, -np.inf])])
    x = x.astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    got = bf16_round(x)
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    assert np.isnan(bf16_round(np.float32([np.nan]))[0])


def test_muon_step_composes_the_steps():
    rng = np.random.default_rng(4)
    W = rng.standard_normal((12, 5)) * 0.02
    g = rng.standard_normal((12, 5)) * 0.01
    buf = rng.standard_normal((12, 5)) * 0.01
    W2, nb, O = muon.muon_step(W, g, buf, beta=0.9, nesterov=True, lr=0.1, wd=0.01)
    nb_ref, u = muon.momentum(g, buf, 0.9, True)
    O_ref = muon.newton_schulz(u)
    assert np.array_equal(nb, nb_ref) and np.array_equal(O, O_ref)
    assert O.shape == (12, 5)
    assert np.allclose(W2, W - 0.1 * 0.01 * W - 0.1 * np.sqrt(12 / 5) * O, rtol=0, atol=1e-15)


# ------------------------------------------------------------------ pair format
# The pair (hi, q) is how the bf16 path carries X between Newton-Schulz steps;
# its definition is the library's (header), restated in oracle/fp32_ref.py.
from fractions import Fraction  # noqa: E402

from oracle.fp32_ref import fma_f32, pair_encode, pair_value  # noqa: E402


def _exponent(hi):
    return int(np.floor(np.log2(abs(float(hi)))))


def test_pair_value_closed_form():
    """value = hi + q 2^(E-15), checked on hand-picked hi (E read off by hand)."""
    hi = np.float32([1.0, 1.5, -0.75, 3.0, 2.0 ** -20])
    q = np.int8([1, -3, 127, -128, 5])
    want = [1.0 + 2.0 ** -15, 1.5 - 3 * 2.0 ** -15, -0.75 + 127 * 2.0 ** -16, 3.0 - 128 * 2.0 ** -14,
            2.0 ** -20 + 5 * 2.0 ** -35]
    assert np.array_equal(pair_value(hi, q), np.array(want))
    # residual unused at 0, for subnormal hi and below 2^-111
    tiny = np.float32([0.0, -0.0, 2.0 ** -130, 2.0 ** -112, 2.0 ** -111])
    got = pair_value(tiny, np.int8([9, 9, 9, 9, 1]))
    assert np.array_equal(got[:4], tiny[:4].astype(np.float64))
    assert got[4] == 2.0 ** -111 + 2.0 ** -126


def test_pair_encode_bound_and_range():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal(50000) * 2.0 ** rng.integers(-60, 60, 50000)).astype(np.float32)
    hi, q = pair_encode(x)
    assert np.array_equal(hi, bf16_round(x))
    err = np.abs(pair_value(hi, q) - x.astype(np.float64))
    E = np.floor(np.log2(np.abs(hi.astype(np.float64))))
    unit = 2.0 ** (E - 15)
    assert np.all(err <= unit)                                      # 2^(E-15) at most (the clamp)
    clamped = (q == 127) & (x.astype(np.float64) - hi > 127.5 * unit)
    assert np.all(err[~clamped] <= unit[~clamped] / 2)              # 2^(E-16) otherwise


def test_pair_encode_round_trips_every_residual():
    """Brute force: for a spread of hi and every q whose value still rounds to
    hi (not at a bf16 tie), encoding the value gives back exactly (hi, q)."""
    rng = np.random.default_rng(6)
    his = bf16_round((rng.standard_normal(64) * 2.0 ** rng.integers(-30, 30, 64)).astype(np.float32))
    his = np.concatenate([his, np.float32([1.0, -2.0, 0.5, 1.0078125])])
    for h in his:
        qs = np.arange(-128, 128, dtype=np.int64)
        v = pair_value(np.full(qs.shape, h, np.float32), qs)
        v32 = v.astype(np.float32)
        assert np.array_equal(v32.astype(np.float64), v)             # exact in fp32
        keep = bf16_round(v32) == h
        # a value exactly halfway to a neighbouring bf16 is a tie the encoder may
        # round either way: leave those out
        bits = int(np.float32(h).view(np.uint32)) >> 16
        nb = np.array([(bits - 1) << 16, (bits + 1) << 16], dtype=np.uint32).view(np.float32)
        mids = (nb.astype(np.float64) + float(h)) / 2.0
        keep &= (v != mids[0]) & (v != mids[1])
        hh, qq = pair_encode(v32[keep])
        assert np.all(hh == h)
        assert np.array_equal(qq.astype(np.int64), qs[keep]), float(h)


def _round_fraction_f32(v):
    """Nearest-even float32 of an exact rational (normal range), by integers only."""
    if v == 0:
        return 0.0
    sign = -1 if v < 0 else 1
    v = abs(v)
    e = v.numerator.bit_length() - v.denominator.bit_length()
    while Fraction(2) ** e > v:
        e -= 1
    while Fraction(2) ** (e + 1) <= v:
        e += 1
    t = v * Fraction(2) ** (23 - e)                  # in [2^23, 2^24)
    n = t.numerator // t.denominator
    rest = t - n
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return sign * float(Fraction(n) * Fraction(2) ** (e - 23))


def test_fma_f32_hand_worked_ties():
    """a x + c exactly halfway between two float32 values except for a tail
    below float64's reach: the tail decides the rounding."""
    one_m = np.float32(1 - 2.0 ** -24)   # a = 1 + 2^-23, x = 1 - 2^-24: a x = 1 + 2^-24 - 2^-47
    a = np.float32(1 + 2.0 ** -23)
    up = np.float32(2.0 ** -47 * (1 + 2.0 ** -23))    # exact sum 1 + 2^-24 + 2^-70: rounds up
    down = np.float32(2.0 ** -47 * (1 - 2.0 ** -24))  # exact sum 1 + 2^-24 - 2^-71: rounds down
    assert fma_f32(a, one_m, up) == np.float32(1 + 2.0 ** -23)
    assert fma_f32(a, one_m, down) == np.float32(1.0)
    # a plain tie (no tail) goes to even
    assert fma_f32(np.float32(1.0), np.float32(1 + 2.0 ** -23), np.float32(2.0 ** -24)) == np.float32(1 + 2.0 ** -22)
    assert fma_f32(np.float32(1.0), np.float32(1.0), np.float32(2.0 ** -24)) == np.float32(1.0)
    # a single product is numpy's float32 multiply
    assert fma_f32(np.float32(3.4445), np.float32(0.3), np.float32(0.0)) == np.float32(3.4445) * np.float32(0.3)


def test_fma_f32_against_exact_rationals():
    rng = np.random.default_rng(7)
    n = 3000
    a = (rng.standard_normal(n) * 2.0 ** rng.integers(-8, 8, n)).astype(np.float32)
    x = (rng.standard_normal(n) * 2.0 ** rng.integers(-8, 8, n)).astype(np.float32)
    c = (rng.standard_normal(n) * 2.0 ** rng.integers(-40, 8, n)).astype(np.float32)
    # near-cancelling and near-tie triples as well
    c[:500] = -(a[:500].astype(np.float64) * x[:500]).astype(np.float32)
    got = fma_f32(a, x, c)
    for i in range(n):
        want = _round_fraction_f32(Fraction(float(a[i])) * Fraction(float(x[i])) + Fraction(float(c[i])))
        assert float(got[i]) == want, (i, a[i], x[i], c[i])
