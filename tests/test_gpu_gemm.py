"""Tensor-core stage kernels against plain fp64 products of the same bf16 values.

Each stage (A = X X^T, B = bA + cA^2, X' = aX + BX) is called through the C ABI
and compared element by element with torch's fp64 CPU product of the very same
operands.  Bounds: bf16 output rounding (2^-8 relative) plus fp32 accumulation
(2^-16 of the sum of absolute products); the symmetric outputs must be exactly
symmetric, and the bf16 copy of X' must be the round-to-nearest of its fp32 value.
"""
import pytest
import torch

import newton_schulz_12_b200 as nsb

pytestmark = pytest.mark.gpu

DEV = "cuda"


def rnd_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g) * scale).to(torch.bfloat16)


def check_close(got, ref, absref, rel=2.0 ** -8, acc=2.0 ** -16):
    got = got.double()
    bound = rel * ref.abs() + acc * absref + 1e-30
    err = (got - ref).abs()
    bad = err > bound
    assert not bad.any(), f"{int(bad.sum())} elements out of bound; worst {float((err - bound).max())}"


# the last cases give every CTA several tiles (persistent loop, both accumulators)
@pytest.mark.parametrize("batch,m,k", [(1, 128, 64), (2, 256, 320), (3, 200, 328), (1, 8, 8),
                                       (2, 768, 3072), (5, 384, 768), (1, 136, 24), (1, 1024, 200),
                                       (160, 256, 136), (40, 768, 768)])
def test_gram(batch, m, k):
    X = rnd_bf16((batch, m, k), seed=m * 7 + k)
    A = nsb.muon_gram_bf16(X.to(DEV)).cpu()
    Xd = X.double()
    ref = Xd @ Xd.transpose(1, 2)
    absref = Xd.abs() @ Xd.abs().transpose(1, 2)
    check_close(A, ref, absref)
    assert torch.equal(A, A.transpose(1, 2)), "A must be exactly symmetric"


@pytest.mark.parametrize("batch,m", [(1, 128), (2, 200), (3, 768), (1, 8), (2, 392), (1, 1024),
                                     (170, 200), (40, 768)])
def test_poly(batch, m):
    G = torch.randn(batch, m, m, generator=torch.Generator().manual_seed(m)) / m ** 0.5
    A = ((G + G.transpose(1, 2)) / 2).to(torch.bfloat16)
    assert torch.equal(A, A.transpose(1, 2))
    b, c = -4.7750, 2.0315
    B = nsb.muon_poly_bf16(A.to(DEV), b, c).cpu()
    Ad = A.double()
    b32, c32 = float(torch.tensor(b, dtype=torch.float32)), float(torch.tensor(c, dtype=torch.float32))
    ref = b32 * Ad + c32 * (Ad @ Ad)
    absref = abs(b32) * Ad.abs() + abs(c32) * (Ad.abs() @ Ad.abs())
    check_close(B, ref, absref)
    assert torch.equal(B, B.transpose(1, 2)), "B must be exactly symmetric"


def pair_unit(hi):
    """2^(E - 15) for hi = 1.f * 2^E (0 where the low part is unused: hi = 0,
    subnormal or below 2^-111), in fp64."""
    h = hi.double()
    _, e = torch.frexp(hi.float())
    E = (e - 1).double()
    ok = (h != 0) & (E >= -111)
    return torch.where(ok, torch.exp2(E - 15), torch.zeros_like(h))


def pair_split(X):
    """The pair format of the iteration: hi = bf16(X), q = nearest-even of
    (X - hi) / 2^(E-15), clamped to [-128, 127] (X fp32, so X - hi is exact)."""
    hi = X.to(torch.bfloat16)
    unit = pair_unit(hi)
    d = X.double() - hi.double()
    q = torch.where(unit > 0, torch.round(d / torch.where(unit > 0, unit, torch.ones_like(unit))),
                    torch.zeros_like(d)).clamp(-128, 127)
    return hi, q.to(torch.int8)


def pair_value(hi, q):
    return hi.double() + q.double() * pair_unit(hi)


def test_pair_format_resolution():
    """The pair holds fp32 values to 2^-16 of |hi|, 2^-15 in the clamped tie
    (CPU check of the test's own encoder)."""
    X = torch.randn(4096, generator=torch.Generator().manual_seed(0)) * torch.exp2(
        torch.randint(-60, 60, (4096,), generator=torch.Generator().manual_seed(1)).float())
    hi, q = pair_split(X)
    err = (pair_value(hi, q) - X.double()).abs()
    assert torch.all(err <= 2.0 ** -15 * hi.double().abs())


# n a multiple of 16 (16-byte rows of the int8 part); 336, 528, 80 leave a ragged 64-column chunk
@pytest.mark.parametrize("batch,m,n", [(1, 128, 128), (2, 200, 336), (1, 768, 3072), (3, 8, 80),
                                       (2, 384, 384), (1, 136, 528), (1, 1024, 4096),
                                       (80, 256, 528), (6, 768, 3072)])
def test_bx(batch, m, n):
    """X' = aX + BX with X carried as the pair (bf16 hi, int8 lo): the output
    pair must hold X' to about 2^-16 and hi' must be bf16(X')."""
    B = rnd_bf16((batch, m, m), seed=m, scale=m ** -0.5)
    X = torch.randn(batch, m, n, generator=torch.Generator().manual_seed(n)) / n ** 0.5
    hi, lo = pair_split(X)
    Xd = pair_value(hi, lo)                  # the X the kernel sees
    a = 3.4445
    a32 = float(torch.tensor(a, dtype=torch.float32))
    lo_dev = lo.cuda()
    hi_out = nsb.muon_bx_bf16(B.cuda(), hi.cuda(), lo_dev, a).cpu()
    lo_out = lo_dev.cpu()
    assert nsb.muon_get_status() == 0
    got = pair_value(hi_out, lo_out)
    ref = a32 * Xd + B.double() @ hi.double()
    absref = abs(a32) * Xd.abs() + B.double().abs() @ hi.double().abs()
    check_close(got, ref, absref, rel=2.0 ** -15, acc=2.0 ** -16)
    # hi' is the round-to-nearest bf16 of X'
    xh = hi_out.double()
    assert torch.all((got - xh).abs() <= 2.0 ** -8 * xh.abs() + 1e-30)


def test_stage_kernels_are_deterministic():
    X = rnd_bf16((4, 768, 3072), seed=1).to(DEV)
    A1 = nsb.muon_gram_bf16(X)
    A2 = nsb.muon_gram_bf16(X)
    assert torch.equal(A1, A2)
    B1 = nsb.muon_poly_bf16(A1)
    B2 = nsb.muon_poly_bf16(A1)
    assert torch.equal(B1, B2)
    assert nsb.muon_get_status() == 0
