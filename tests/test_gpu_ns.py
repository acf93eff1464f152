"""muon_ns_orthogonalize (C ABI) against the fp64 oracle on the same inputs.

bf16 mode: relative Frobenius error <= 3e-2 (bf16 tensor-core operands, fp32
accumulation); fp32 mode: <= 1e-4 (fp32 SIMT FMA).  The oracle receives the
exact values the GPU receives (bf16 inputs are widened exactly).
"""
import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from blockcheck import assert_blocks
from newton_schulz_12_b200 import workloads
from oracle import muon as oracle

pytestmark = pytest.mark.gpu

TOL_BF16 = 3e-2
TOL_FP32 = 1e-4
# every 32 x 32 block within 4x the whole-matrix bound (tests/blockcheck.py)
BLOCK_TOL_BF16 = 4 * TOL_BF16
BLOCK_TOL_FP32 = 4 * TOL_FP32


def rel_fro(got, ref):
    got = np.asarray(got, dtype=np.float64)
    return np.linalg.norm(got - ref) / np.linalg.norm(ref)


def run_ns(mats, steps=5, coeffs=oracle.NS_COEFFS):
    dev = [m.clone().cuda() for m in mats]
    nsb.muon_ns_orthogonalize(dev, *coeffs, steps=steps)
    assert nsb.muon_get_status() == 0
    return [d.float().cpu().numpy() for d in dev]


def test_config1_single_768_fp32_and_bf16():
    """768x768 fp32, iid N(0,1) from seed 0, T=5, in both modes."""
    X = workloads.gaussian((768, 768), 1.0, seed=0)
    ref = oracle.newton_schulz(X.double().numpy())
    got32 = run_ns([X])[0]
    assert rel_fro(got32, ref) <= TOL_FP32
    assert_blocks(got32, ref, BLOCK_TOL_FP32, "fp32 768x768")
    Xb = X.to(torch.bfloat16)
    ref_b = oracle.newton_schulz(Xb.double().numpy())
    got16 = run_ns([Xb])[0]
    assert rel_fro(got16, ref_b) <= TOL_BF16
    assert_blocks(got16, ref_b, BLOCK_TOL_BF16, "bf16 768x768")


@pytest.mark.parametrize("rows,cols,batch", [
    (768, 768, 2), (768, 3072, 2), (3072, 768, 1), (200, 328, 3), (328, 200, 2), (130, 390, 1),
    (8, 8, 4), (1, 17, 1), (17, 1, 1), (1, 1, 2), (64, 1000, 1), (1024, 1024, 1), (256, 4096, 1)])
def test_bf16_shapes(rows, cols, batch):
    mats = [workloads.gaussian((rows, cols), 1.0, seed=100 + i, dtype=torch.bfloat16)
            for i in range(batch)]
    got = run_ns(mats)
    for g, x in zip(got, mats):
        assert g.shape == (rows, cols)
        ref = oracle.newton_schulz(x.double().numpy())
        assert rel_fro(g, ref) <= TOL_BF16
        assert_blocks(g, ref, BLOCK_TOL_BF16, f"{rows}x{cols}")


@pytest.mark.parametrize("rows,cols", [(768, 3072), (200, 328), (328, 200), (8, 8), (1, 5), (96, 96)])
def test_fp32_shapes(rows, cols):
    X = workloads.gaussian((rows, cols), 1.0, seed=rows + cols)
    got = run_ns([X])[0]
    ref = oracle.newton_schulz(X.double().numpy())
    assert rel_fro(got, ref) <= TOL_FP32
    assert_blocks(got, ref, BLOCK_TOL_FP32, f"fp32 {rows}x{cols}")


@pytest.mark.parametrize("steps", [0, 1, 2, 7])
def test_step_counts(steps):
    X = workloads.gaussian((384, 640), 1.0, seed=steps, dtype=torch.bfloat16)
    ref = oracle.newton_schulz(X.double().numpy(), steps=steps)
    assert rel_fro(run_ns([X], steps=steps)[0], ref) <= TOL_BF16
    X32 = X.float()
    assert rel_fro(run_ns([X32], steps=steps)[0], ref) <= TOL_FP32


def test_other_coefficients():
    """A different (a, b, c): the classic cubic 1.5 X - 0.5 X X^T X."""
    X = workloads.gaussian((256, 512), 1.0, seed=3, dtype=torch.bfloat16)
    coeffs = (1.5, -0.5, 0.0)
    ref = oracle.newton_schulz(X.double().numpy(), steps=5, coeffs=coeffs)
    assert rel_fro(run_ns([X], steps=5, coeffs=coeffs)[0], ref) <= TOL_BF16


@pytest.mark.parametrize("scale", [2.0 ** 60, 2.0 ** 45, 2.0 ** -45, 2.0 ** -100])
def test_bf16_extreme_magnitudes(scale):
    """Norms far from 1: the first Gram product runs on the unnormalised pair,
    so norms beyond 2^40 are rescaled by a power of two first and tiny inputs
    reduce to X_k ~ a^k X0 (A underflows), as in the oracle."""
    X = (workloads.gaussian((256, 640), 1.0, seed=11) * scale).to(torch.bfloat16)
    ref = oracle.newton_schulz(X.double().numpy())
    got = run_ns([X])[0]
    assert np.all(np.isfinite(got))
    assert rel_fro(got, ref) <= TOL_BF16


@pytest.mark.parametrize("rows,cols,batch", [(1, 32768, 1), (32768, 1, 1), (8, 32768, 2)])
def test_maximum_dimension(rows, cols, batch):
    """The largest side the ABI accepts (32768): a single row / column is
    normalised and stays a unit vector scaled by the chained scalar map."""
    mats = [workloads.gaussian((rows, cols), 1.0, seed=900 + i, dtype=torch.bfloat16)
            for i in range(batch)]
    got = run_ns(mats)
    for g, x in zip(got, mats):
        assert rel_fro(g, oracle.newton_schulz(x.double().numpy())) <= TOL_BF16


def test_rank_one_and_constant_matrices():
    """All the mass in one singular value (sigma = 1 after normalisation):
    rank-1 outer products and an all-equal matrix follow p(p(...p(1)))."""
    g = torch.Generator().manual_seed(12)
    u = torch.randn(384, 1, generator=g)
    v = torch.randn(1, 640, generator=g)
    for X in ((u @ v).to(torch.bfloat16), torch.full((256, 512), 0.5).to(torch.bfloat16)):
        ref = oracle.newton_schulz(X.double().numpy())
        assert rel_fro(run_ns([X])[0], ref) <= TOL_BF16


def test_zero_matrix_gives_zero():
    for dt in (torch.bfloat16, torch.float32):
        got = run_ns([torch.zeros(64, 96, dtype=dt)])[0]
        assert np.all(got == 0.0)


def test_hard_spectrum_band():
    """Log-uniform spectrum with a x100 spike: still within tolerance of the oracle."""
    G = workloads.hard_spectrum(768, 768, seed=5, spike=True)
    ref = oracle.newton_schulz(G.double().numpy())
    got = run_ns([G])[0]
    assert rel_fro(got, ref) <= TOL_BF16
    assert_blocks(got, ref, BLOCK_TOL_BF16, "hard spectrum")


def test_deterministic():
    X = workloads.gaussian((768, 3072), 1.0, seed=9, dtype=torch.bfloat16)
    a = run_ns([X])[0]
    b = run_ns([X])[0]
    assert np.array_equal(a, b)


@pytest.mark.parametrize("rows,cols,batch", [(64, 192, 168), (40, 100, 3), (300, 1000, 2)])
def test_last_step_writes_outputs_directly_or_through_the_pass(rows, cols, batch):
    """The last BX launch stores X_T (rounded to bf16) straight into the
    callers' buffers for the first 160 matrices of a launch whose rows are
    16-byte strided; the rest (past the table, or cols % 8 != 0) go through
    the write-back pass.  Every output is checked against the oracle."""
    mats = [workloads.gaussian((rows, cols), 1.0, seed=7300 + i, dtype=torch.bfloat16)
            for i in range(batch)]
    got = run_ns(mats)
    for i in range(batch):
        ref = oracle.newton_schulz(mats[i].double().numpy())
        assert rel_fro(got[i], ref) <= TOL_BF16, i
        assert_blocks(got[i], ref, BLOCK_TOL_BF16, f"matrix {i}")


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_non_finite_matrix_leaves_the_others_unchanged(bad):
    """Matrices are independent (the iteration is per matrix): a NaN or an inf
    in one matrix of a batch changes no bit of the other matrices' results,
    so no reduction, tile or table entry mixes them."""
    mats = [workloads.gaussian((300, 1000), 1.0, seed=7500 + i, dtype=torch.bfloat16) for i in range(4)]
    clean = run_ns(mats)
    dirty = [m.clone() for m in mats]
    dirty[1][5, 7] = bad
    got = run_ns(dirty)
    for i in (0, 2, 3):
        assert np.array_equal(got[i], clean[i]), i
