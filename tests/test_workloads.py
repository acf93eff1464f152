"""The seeded input recipe (shared by the tests, the benchmark and the oracle
legs) against its stated definition: shapes, batch sizes, seeds, and the
spectra of the hard-spectrum gradients."""
import numpy as np
import pytest
import torch

from newton_schulz_12_b200 import workloads


def test_square_sweep_batches():
    assert workloads.sweep_cases() == [(256, 576), (512, 144), (768, 64), (1024, 36), (2048, 9),
                                       (4096, 2)]


def test_scaled_set_is_144_matrices_1024_wide():
    s = workloads.scaled_shapes()
    assert len(s) == 144 and s[:6] == [(1024, 1024)] * 4 + [(1024, 4096), (4096, 1024)]


def test_gaussian_is_seeded_and_cast_after_an_fp32_draw():
    a = workloads.gaussian((64, 48), 0.5, seed=11)
    b = workloads.gaussian((64, 48), 0.5, seed=11)
    assert torch.equal(a, b) and a.dtype == torch.float32
    assert not torch.equal(a, workloads.gaussian((64, 48), 0.5, seed=12))
    h = workloads.gaussian((64, 48), 0.5, seed=11, dtype=torch.bfloat16)
    assert torch.equal(h, a.to(torch.bfloat16))
    big = workloads.gaussian((512, 512), 0.01, seed=3).double()
    assert float(big.std()) == pytest.approx(0.01, rel=0.02)
    assert abs(float(big.mean())) < 1e-4


@pytest.mark.parametrize("rows,cols", [(96, 160), (160, 96)])
def test_hard_spectrum_singular_values(rows, cols):
    G = workloads.hard_spectrum(rows, cols, seed=5, dtype=torch.float32).double().numpy()
    s = np.linalg.svd(G, compute_uv=False)
    k = min(rows, cols)
    assert s.shape == (k,)
    # log-uniform in [1e-4, 1] times scale 1e-2, up to the fp32 cast
    assert s.max() <= 1e-2 * (1 + 1e-5) and s.min() >= 1e-6 * (1 - 1e-3)
    logs = np.log10(s / 1e-2)
    assert -4.0 - 1e-3 <= logs.min() and logs.max() <= 1e-5
    # roughly uniform in the exponent: each quarter of [-4, 0] holds about a quarter
    counts = np.histogram(logs, bins=4, range=(-4, 0))[0]
    assert counts.min() >= k // 8


def test_hard_spectrum_spike():
    plain = workloads.hard_spectrum(80, 120, seed=9, dtype=torch.float32).double().numpy()
    spiked = workloads.hard_spectrum(80, 120, seed=9, spike=True, dtype=torch.float32).double().numpy()
    sp = np.linalg.svd(plain, compute_uv=False)
    ss = np.linalg.svd(spiked, compute_uv=False)
    np.testing.assert_allclose(ss[:4], 100 * sp[:4], rtol=1e-5)
    np.testing.assert_allclose(ss[4:], sp[4:], rtol=1e-4, atol=1e-9)


def test_spiked_indices_for_the_72_matrix_set():
    idx = workloads.spiked_indices(72)
    assert len(idx) == 4 and len(set(idx)) == 4 and all(0 <= i < 72 for i in idx)
    assert workloads.spiked_indices(72) == idx


def test_muon_set_seeds():
    shapes = [(16, 24), (24, 16), (8, 8)]
    Ws, Gs = workloads.muon_set(shapes, step=2)
    for i, s in enumerate(shapes):
        assert torch.equal(Ws[i], workloads.gaussian(s, 2e-2, 2000 + i))
        assert torch.equal(Gs[i], workloads.gaussian(s, 1e-2, 1000 + i + 200, torch.bfloat16))
        assert Ws[i].dtype == torch.float32 and Gs[i].dtype == torch.bfloat16
    Ws0, Gs0 = workloads.muon_set(shapes, step=0)
    assert all(torch.equal(a, b) for a, b in zip(Ws, Ws0))   # W does not depend on the step
    assert not any(torch.equal(a, b) for a, b in zip(Gs, Gs0))
