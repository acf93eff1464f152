"""Stray writes into caller memory: every buffer the library writes lies inside
one larger allocation filled with a sentinel byte, with 4 KiB gaps around and
between the buffers (and, for the stage call with padded rows, the padding
columns).  After each call every byte outside the buffers' own elements must
still hold the sentinel.

The last Newton-Schulz launch stores straight into caller memory with bulk
tensor copies (W in muon_step, the outputs of the NS-only calls), so an
out-of-range row or column at a ragged edge would land in a neighbouring
tensor; this is the check that would see it.
"""
import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import workloads

pytestmark = pytest.mark.gpu

GAP = 4096
SENTINEL = 0xA5


class Arena:
    """Tensors carved out of one sentinel-filled byte buffer with GAP bytes around each."""

    def __init__(self, specs):
        sizes = [int(np.prod(shape)) * torch.empty(0, dtype=dt).element_size() for shape, dt in specs]
        offs, off = [], GAP
        for sz in sizes:
            offs.append(off)
            off += (sz + 255) // 256 * 256 + GAP
        self.buf = torch.full((off,), SENTINEL, dtype=torch.uint8, device="cuda")
        self.spans = list(zip(offs, sizes))
        self.tensors = [self.buf[o:o + sz].view(dt).view(shape)
                        for (o, sz), (shape, dt) in zip(self.spans, specs)]

    def check(self, what=""):
        mask = torch.ones_like(self.buf, dtype=torch.bool)
        for o, sz in self.spans:
            mask[o:o + sz] = False
        bad = (self.buf != SENTINEL) & mask
        n = int(bad.sum())
        assert n == 0, f"{what}: {n} sentinel bytes overwritten, first at {int(bad.nonzero()[0])}"


SHAPES = [(768, 3072), (3072, 768), (130, 68), (68, 130), (77, 5), (5, 77), (1, 40), (40, 1), (200, 328)]


def test_muon_step_writes_only_its_buffers():
    specs = []
    for s in SHAPES:
        specs += [(s, torch.float32), (s, torch.bfloat16), (s, torch.float32)]
    ar = Arena(specs)
    Ws, Gs = workloads.muon_set(SHAPES, step=0)
    for i in range(len(SHAPES)):
        ar.tensors[3 * i].copy_(Ws[i])
        ar.tensors[3 * i + 1].copy_(Gs[i])
        ar.tensors[3 * i + 2].zero_()
    for step in range(2):
        nsb.muon_step(ar.tensors[0::3], ar.tensors[1::3], ar.tensors[2::3], wd=0.01)
        assert nsb.muon_get_status() == 0
        ar.check(f"muon_step {step}")
    # the refinements take the apply pass for every matrix
    V = Arena([((s[0],), torch.float32) for s in SHAPES])
    for v in V.tensors:
        v.zero_()
    nsb.muon_step_ex(ar.tensors[0::3], ar.tensors[1::3], ar.tensors[2::3], wd=0.01, cautious_wd=True,
                     neuron_state=V.tensors)
    assert nsb.muon_get_status() == 0
    ar.check("muon_step_ex")
    V.check("neuron state")


def test_table_overflow_writes_only_its_buffers():
    """168 matrices: 160 through the fused epilogue, 8 through the apply pass."""
    shapes = [(64, 192), (192, 64)] * 84
    specs = []
    for s in shapes:
        specs += [(s, torch.float32), (s, torch.bfloat16), (s, torch.float32)]
    ar = Arena(specs)
    Ws, Gs = workloads.muon_set(shapes, step=0)
    for i in range(len(shapes)):
        ar.tensors[3 * i].copy_(Ws[i])
        ar.tensors[3 * i + 1].copy_(Gs[i])
        ar.tensors[3 * i + 2].zero_()
    nsb.muon_step(ar.tensors[0::3], ar.tensors[1::3], ar.tensors[2::3], wd=0.5)
    assert nsb.muon_get_status() == 0
    ar.check("overflow step")


@pytest.mark.parametrize("rows,cols,batch", [(768, 3072, 2), (3072, 768, 1), (130, 68, 3), (68, 136, 3),
                                             (64, 192, 168), (5, 77, 2)])
def test_ns_writes_only_its_buffers(rows, cols, batch):
    """Direct write-back by the last GEMM (wide, 16-byte rows, first 160) and
    the write-back pass (tall, ragged, past the table)."""
    ar = Arena([((rows, cols), torch.bfloat16)] * batch)
    for i, t in enumerate(ar.tensors):
        t.copy_(workloads.gaussian((rows, cols), 1.0, seed=60 + i, dtype=torch.bfloat16))
    nsb.muon_ns_orthogonalize(ar.tensors)
    assert nsb.muon_get_status() == 0
    ar.check(f"ns {rows}x{cols}")


def test_stage_calls_write_only_their_buffers():
    """The fused last step with padded rows (ldx 160 for n = 130): Xhi and its
    padding are read only; the tall (fused) matrix's Xlo is read only; the
    matrices that take the separate pass get q of X' in Xlo, written in whole
    16-byte units, so columns 130 .. 143 may change and 144 .. 159 may not."""
    m, n, ldx, ldb = 68, 130, 160, 72
    ar = Arena([((3, m, ldb), torch.bfloat16), ((3, m, ldx), torch.bfloat16), ((3, m, ldx), torch.int8),
                ((n, m), torch.float32), ((m, n), torch.float32), ((m, n), torch.float32)])
    B, hi, lo, W0, W1, W2 = ar.tensors
    g = torch.Generator(device="cpu").manual_seed(5)
    B.copy_((torch.randn(3, m, ldb, generator=g) * 0.05).to(torch.bfloat16))
    hi.copy_((torch.randn(3, m, ldx, generator=g) * 0.1).to(torch.bfloat16))
    lo.copy_(torch.randint(-128, 128, (3, m, ldx), generator=g, dtype=torch.int8))
    # the padding columns of the operands hold random values
    hi0 = hi.clone()
    lo0 = lo.clone()
    n16 = (n + 15) // 16 * 16
    for w in (W0, W1, W2):
        w.copy_(torch.randn(w.shape, generator=g) * 0.02)
    # one call per layout: tall W (n x m), and two wide W whose columns are not
    # a multiple of 4 (the pass)
    nsb.muon_bx_apply_bf16(B[:1], hi[:1], lo[:1], [W0], n=n, tall=True, wd=0.1)
    nsb.muon_bx_apply_bf16(B[1:], hi[1:], lo[1:], [W1, W2], n=n, tall=False, wd=0.1, cautious=True)
    assert nsb.muon_get_status() == 0
    ar.check("bx_apply")
    assert torch.equal(hi, hi0)
    assert torch.equal(lo[0], lo0[0])
    assert torch.equal(lo[1:, :, n16:], lo0[1:, :, n16:])
