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
