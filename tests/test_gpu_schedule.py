"""muon_ns_orthogonalize_schedule (one (a, b, c) per step) against the oracle.

"The NanoGPT speedrun", paragraph "Reading guide", names Polar Express
polynomials: the same iteration with per-step coefficients.  The pages print
none, so the schedules here are triples chosen for the test (the speedrun
quintic, the classic cubic, the flat quintic 15/8, -10/8, 3/8).  Tolerances
as for the fixed triple: 3e-2 relative Frobenius (bf16 path), 1e-4 (fp32).
"""
import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import workloads
from oracle import muon as oracle

pytestmark = pytest.mark.gpu

QUINTIC = (3.4445, -4.7750, 2.0315)
CUBIC = (1.5, -0.5, 0.0)
FLAT = (15 / 8, -10 / 8, 3 / 8)


def f32(t):
    """The triple as the library receives it (fp32)."""
    return tuple(float(np.float32(v)) for v in t)


def rel_fro(got, ref):
    got = np.asarray(got, dtype=np.float64)
    return np.linalg.norm(got - ref) / np.linalg.norm(ref)


def run(mats, schedule):
    dev = [m.clone().cuda() for m in mats]
    nsb.muon_ns_orthogonalize_schedule(dev, schedule)
    assert nsb.muon_get_status() == 0
    return [d.float().cpu().numpy() for d in dev]


@pytest.mark.parametrize("rows,cols,batch,dtype", [
    (768, 3072, 2, torch.bfloat16), (3072, 768, 1, torch.bfloat16), (200, 328, 3, torch.bfloat16),
    (768, 768, 2, torch.bfloat16), (200, 328, 1, torch.float32), (96, 64, 2, torch.float32)])
def test_schedule_matches_oracle(rows, cols, batch, dtype):
    schedule = [QUINTIC, QUINTIC, CUBIC, FLAT, CUBIC, FLAT]
    mats = [workloads.gaussian((rows, cols), 1.0, seed=700 + i, dtype=dtype) for i in range(batch)]
    got = run(mats, schedule)
    tol = 3e-2 if dtype == torch.bfloat16 else 1e-4
    for g, x in zip(got, mats):
        ref = oracle.newton_schulz(x.double().numpy(), schedule=[f32(t) for t in schedule])
        assert rel_fro(g, ref) <= tol


def test_constant_schedule_equals_the_fixed_triple_call():
    X = workloads.gaussian((768, 3072), 1.0, seed=9, dtype=torch.bfloat16)
    a = run([X], [QUINTIC] * 5)[0]
    b = X.clone().cuda()
    nsb.muon_ns_orthogonalize([b], *QUINTIC, steps=5)
    assert np.array_equal(a, b.float().cpu().numpy())


def test_order_of_the_schedule_matters_on_the_gpu():
    """Forward and reversed schedules are different functions; the GPU follows
    the order given (each result matches its own oracle, not the other's)."""
    # three quintic steps first take the singular values into the nonlinear
    # range; reversed, the cubic and flat steps act while they are still small
    schedule = [QUINTIC, QUINTIC, QUINTIC, CUBIC, FLAT]
    X = workloads.hard_spectrum(256, 512, seed=4, spike=False).to(torch.bfloat16)
    fwd = run([X], schedule)[0]
    rev = run([X], schedule[::-1])[0]
    ref_f = oracle.newton_schulz(X.double().numpy(), schedule=[f32(t) for t in schedule])
    ref_r = oracle.newton_schulz(X.double().numpy(), schedule=[f32(t) for t in schedule[::-1]])
    assert rel_fro(fwd, ref_f) <= 3e-2 and rel_fro(rev, ref_r) <= 3e-2
    assert rel_fro(ref_f, ref_r) > 0.1


def test_empty_schedule_normalises():
    X = workloads.gaussian((128, 256), 1.0, seed=5, dtype=torch.bfloat16)
    got = run([X], [])[0]
    ref = oracle.newton_schulz(X.double().numpy(), schedule=[])
    assert rel_fro(got, ref) <= 1e-2


def test_schedule_on_a_tall_hard_spectrum():
    """Transposed (tall) input with a log-uniform spectrum through a mixed schedule."""
    schedule = [QUINTIC, QUINTIC, FLAT, QUINTIC, CUBIC]
    X = workloads.hard_spectrum(1024, 384, seed=8, spike=True)
    got = run([X], schedule)[0]
    ref = oracle.newton_schulz(X.double().numpy(), schedule=[f32(t) for t in schedule])
    assert rel_fro(got, ref) <= 3e-2
