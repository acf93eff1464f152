"""Checkpoint / resume and the square width sweep.

The library is stateless: the caller owns weights and momentum buffers.  k
steps, a save to host and a reload, then one more step must equal k+1
uninterrupted steps bit for bit (fixed reduction orders, no atomics).
The width sweep runs m in {256..4096} square matrices, batch 64*(768/m)^2,
against the fp64 oracle, every matrix of every width (whole-matrix relative
Frobenius error and every 32 x 32 block).
"""
import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from blockcheck import assert_blocks
from newton_schulz_12_b200 import workloads
from oracle import muon as oracle

pytestmark = pytest.mark.gpu


def run_steps(W, M, shapes, first, last):
    for step in range(first, last):
        _, Gs = workloads.muon_set(shapes, step=step)
        nsb.muon_step(W, [g.cuda() for g in Gs], M, wd=0.01)
    assert nsb.muon_get_status() == 0


def test_resume_is_bit_exact():
    shapes = [(768, 768), (768, 3072), (3072, 768), (200, 328)]
    Ws, _ = workloads.muon_set(shapes)
    W1 = [w.cuda() for w in Ws]
    M1 = [torch.zeros(s, device="cuda") for s in shapes]
    run_steps(W1, M1, shapes, 0, 3)
    # checkpoint to host, resume in fresh tensors
    ck = {"W": [w.cpu().clone() for w in W1], "M": [m.cpu().clone() for m in M1]}
    W2 = [w.cuda() for w in ck["W"]]
    M2 = [m.cuda() for m in ck["M"]]
    run_steps(W1, M1, shapes, 3, 4)
    run_steps(W2, M2, shapes, 3, 4)
    for a, b in zip(W1 + M1, W2 + M2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("m,batch", workloads.sweep_cases())
def test_width_sweep(m, batch):
    xs = [workloads.gaussian((m, m), 1.0, seed=3000 + m + i, dtype=torch.bfloat16) for i in range(batch)]
    dev = [x.cuda() for x in xs]
    nsb.muon_ns_orthogonalize(dev)
    assert nsb.muon_get_status() == 0
    for i in range(batch):
        ref = oracle.newton_schulz(xs[i].double().numpy())
        got = dev[i].double().cpu().numpy()
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert err <= 3e-2, (m, i, err)
        assert_blocks(got, ref, 4 * 3e-2, f"m = {m}, matrix {i}")
