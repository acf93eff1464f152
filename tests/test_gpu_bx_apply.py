"""The last Newton-Schulz product with the apply fused into it, bit for bit.

muon_step applies most updates inside its last GEMM launch (the "then scaled
and applied" of "The NanoGPT speedrun", record #3).  muon_bx_apply_bf16 runs
that launch alone, so W' can be compared bitwise with the fp32 restatement of
the apply (oracle/fp32_ref.apply_f32) given the O the epilogue forms:

* B = 0: the accumulator is exactly 0, O = fl(a * X) with X the pair's exact
  value, one rounding;
* B != 0 on a coarse grid (B = k 2^-6, hi = j 2^-6, small k, j): every partial
  sum of B hi is a multiple of 2^-12 below 2^5, so the fp32 accumulation is
  exact whatever its order and O = fl(a X + B hi) is one rounding of an exact
  value (oracle/fp32_ref.fma_f32);
* matrices past the epilogue's 160-entry table, or whose W has a column count
  that is not a multiple of 4, take the pair write and the apply pass: their
  O is the pair's value of that same fp32 O (oracle/fp32_ref.pair_encode).

Layouts: W in X's layout (wide, square) and W = X^T (tall), ragged sizes
(row strides padded as the workspace pads them), lr * wd != 0, and
cautious weight decay (the decay term only where W * O > 0).
"""
import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from oracle.fp32_ref import apply_f32, fma_f32, pair_encode, pair_value, update_scale_f32

pytestmark = pytest.mark.gpu

A_COEF = np.float32(3.4445)


def _pad(v, k):
    return (v + k - 1) // k * k


def make_case(batch, m, n, seed, grid):
    """Seeded operands: B (batch, m, ldb), the pair (hi, q) of X (batch, m, ldx)."""
    rng = np.random.default_rng(seed)
    ldx, ldb = _pad(n, 16), _pad(m, 8)
    if grid:
        B = rng.integers(-8, 9, (batch, m, ldb)).astype(np.float32) * np.float32(2.0 ** -6)
        hi = rng.integers(-16, 17, (batch, m, ldx)).astype(np.float32) * np.float32(2.0 ** -6)
    else:
        B = np.zeros((batch, m, ldb), np.float32)
        hi = (rng.standard_normal((batch, m, ldx)) / np.sqrt(n)).astype(np.float32)
        hi = torch.from_numpy(hi).to(torch.bfloat16).float().numpy()
    B[:, :, m:] = 0.0
    q = rng.integers(-128, 128, (batch, m, ldx)).astype(np.int8)
    hi[:, :, n:] = 0.0
    q[:, :, n:] = 0
    return B, hi, q, ldx


def expected_O(B, hi, q, m, n):
    """fp32 O = fl(a X + B hi) per matrix (m x n), exact accumulation assumed."""
    X = pair_value(hi[:, :, :n], q[:, :, :n])                      # exact, fits fp32
    acc = np.einsum("bij,bjk->bik", B[:, :, :m].astype(np.float64), hi[:, :, :n].astype(np.float64))
    assert np.array_equal(acc.astype(np.float32).astype(np.float64), acc)  # exactly representable
    return fma_f32(A_COEF, X.astype(np.float32), acc.astype(np.float32))


def run_case(batch, m, n, tall, lr, wd, seed, grid, cautious=False):
    B, hi, q, ldx = make_case(batch, m, n, seed, grid)
    rows, cols = (n, m) if tall else (m, n)
    rng = np.random.default_rng(seed + 1)
    W0 = [(rng.standard_normal((rows, cols)) * 0.02).astype(np.float32) for _ in range(batch)]
    dB = torch.from_numpy(B).to(torch.bfloat16).cuda()
    dhi = torch.from_numpy(hi).to(torch.bfloat16).cuda()
    dq = torch.from_numpy(q).cuda()
    W = [torch.from_numpy(w.copy()).cuda() for w in W0]
    nsb.muon_bx_apply_bf16(dB, dhi, dq, W, n=n, tall=tall, a=float(A_COEF), lr=lr, wd=wd,
                           cautious=cautious)
    assert nsb.muon_get_status() == 0
    O = expected_O(B, hi, q, m, n)
    scale = update_scale_f32(rows, cols)
    for i in range(batch):
        fused = i < 160 and cols % 4 == 0
        Oi = O[i] if fused else pair_value(*pair_encode(O[i])).astype(np.float32)
        ref = apply_f32(W0[i], Oi.T if tall else Oi, lr, wd, scale, cautious=cautious)
        got = W[i].cpu().numpy()
        bad = got.view(np.uint32) != ref.view(np.uint32)
        assert not bad.any(), (f"matrix {i} ({'fused' if fused else 'pass'}): {int(bad.sum())} of "
                               f"{bad.size} elements differ; first at {np.argwhere(bad)[0].tolist()}")


# (batch, m, n, tall): X is m x n; W is m x n, or n x m when tall
LAYOUTS = [
    (2, 768, 3072, False),   # MLP-in: W in X's layout, mode 1
    (2, 768, 3072, True),    # MLP-out: W = X^T, mode 2
    (3, 768, 768, False),    # attention square
    (2, 68, 132, False),     # ragged, 132 columns: a partial 32-column chunk
    (2, 68, 130, True),      # W 130 x 68 (tall, ragged both ways)
    (1, 68, 130, False),     # W 68 x 130: columns not a multiple of 4 -> pass
    (1, 5, 77, True),        # W 77 x 5 -> pass
    (1, 5, 77, False),       # W 5 x 77 -> pass
    (3, 200, 328, True),
]


@pytest.mark.parametrize("batch,m,n,tall", LAYOUTS)
def test_zero_b_bitwise(batch, m, n, tall):
    run_case(batch, m, n, tall, lr=0.05, wd=0.0, seed=m * 31 + n, grid=False)


@pytest.mark.parametrize("batch,m,n,tall", LAYOUTS)
def test_exact_grid_bitwise_with_decay(batch, m, n, tall):
    run_case(batch, m, n, tall, lr=0.05, wd=0.1, seed=m * 17 + n + 1, grid=True)


@pytest.mark.parametrize("batch,m,n,tall", LAYOUTS)
def test_cautious_decay_bitwise(batch, m, n, tall):
    """Cautious weight decay (decay only where W and O share a sign) in the
    fused epilogue and in the pass, lr * wd large enough to matter."""
    run_case(batch, m, n, tall, lr=0.05, wd=2.0, seed=m * 13 + n + 2, grid=True, cautious=True)


def test_weight_decay_dominant():
    run_case(2, 256, 512, False, lr=0.01, wd=20.0, seed=11, grid=True)
    run_case(2, 256, 512, True, lr=0.01, wd=20.0, seed=12, grid=True)


@pytest.mark.parametrize("tall", [False, True])
def test_more_than_the_table(tall):
    """168 matrices in one launch: 160 applied in the epilogue, 8 by the pass."""
    run_case(168, 64, 192, tall, lr=0.05, wd=0.5, seed=13 + tall, grid=True)


def test_rejects_bad_strides():
    x = torch.zeros(1, 8, 24, dtype=torch.bfloat16, device="cuda")
    q = torch.zeros(1, 8, 24, dtype=torch.int8, device="cuda")
    B = torch.zeros(1, 8, 8, dtype=torch.bfloat16, device="cuda")
    W = [torch.zeros(8, 24, device="cuda")]
    with pytest.raises(nsb.MuonError):
        nsb.muon_bx_apply_bf16(B, x, q, W)
