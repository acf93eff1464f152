"""The sharded Muon step on the GPU: one NCCL rank through the product path.

With one rank the group step is the plain muon_step, so the sharded object
(its flat buffers, the in-place reduce-scatter and all-gather on NCCL, the
per-bucket prepared steps) must reproduce muon_step on the same inputs bit
for bit: every matrix's arithmetic is independent of which other matrices
share its launches (no reduction crosses matrices, each output tile is summed
by one CTA pair in a fixed K order, the norm partials per block in a fixed
order), and averaging over one rank leaves the gradients unchanged.  It must
also match the oracle within the step tolerance.  More ranks need more GPUs than one
run has; their host logic is covered on CPU by test_sharded.py.
"""
import socket

import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import workloads
from newton_schulz_12_b200.sharded import ShardedMuon
from oracle import muon as oracle

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_one_nccl_rank_reproduces_muon_step():
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        shapes = workloads.gpt2_small_shapes(layers=2) + [(300, 1000), (77, 5)]
        Ws, Gs = workloads.muon_set(shapes, step=0)
        sm = ShardedMuon(shapes, device="cuda", buckets=3, lr=0.05, wd=0.01)
        for i in range(len(shapes)):
            sm.params[i].copy_(Ws[i])
        W_ref = [w.cuda() for w in Ws]
        M_ref = [torch.zeros_like(w) for w in W_ref]
        for step in range(2):
            _, Gs = workloads.muon_set(shapes, step=step)
            for i in range(len(shapes)):
                sm.grads[i].copy_(Gs[i])
            W0 = [p.cpu().numpy() for p in sm.params]
            M0 = [m.cpu().numpy() for m in sm.momentum]
            sm.step()
            nsb.muon_step(W_ref, [g.cuda() for g in Gs], M_ref, lr=0.05, wd=0.01)
            torch.cuda.synchronize()
            assert nsb.muon_get_status() == 0
            for i, s in enumerate(shapes):
                np.testing.assert_array_equal(sm.momentum[i].cpu().numpy(), M_ref[i].cpu().numpy())
                np.testing.assert_array_equal(sm.params[i].cpu().numpy(), W_ref[i].cpu().numpy())
            for i in (0, 4, 5, len(shapes) - 2):  # against the oracle on the pre-step state
                Wn, _, _ = oracle.muon_step(W0[i], Gs[i].float().numpy(), M0[i],
                                            beta=np.float32(0.95), nesterov=True,
                                            lr=np.float32(0.05), wd=np.float32(0.01))
                dW = sm.params[i].cpu().numpy().astype(np.float64) - W0[i]
                err = np.linalg.norm(dW - (Wn - W0[i])) / np.linalg.norm(Wn - W0[i])
                assert err <= 3e-2, (i, err)
    finally:
        dist.destroy_process_group()


def test_one_nccl_rank_with_refinements_reproduces_muon_step_ex():
    """Cautious decay, NorMuon (state kept by the owner) and a per-step
    schedule through the sharded object: bit for bit muon_step_ex on the same
    inputs, weights, momentum and state."""
    import torch.distributed as dist
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, device_id=torch.device("cuda", 0))
    try:
        shapes = workloads.gpt2_small_shapes(layers=1) + [(300, 1000), (77, 5)]
        sched = [(3.4445, -4.7750, 2.0315)] * 3 + [(15 / 8, -10 / 8, 3 / 8), (1.5, -0.5, 0.0)]
        Ws, _ = workloads.muon_set(shapes, step=0)
        sm = ShardedMuon(shapes, device="cuda", buckets=2, lr=0.05, wd=0.3, cautious_wd=True,
                         normuon=True, beta2=0.9, schedule=sched)
        for i in range(len(shapes)):
            sm.params[i].copy_(Ws[i])
        W_ref = [w.cuda() for w in Ws]
        M_ref = [torch.zeros_like(w) for w in W_ref]
        V_ref = [torch.zeros(w.shape[0], device="cuda") for w in W_ref]
        for step in range(2):
            _, Gs = workloads.muon_set(shapes, step=step)
            for i in range(len(shapes)):
                sm.grads[i].copy_(Gs[i])
            sm.step()
            nsb.muon_step_ex(W_ref, [g.cuda() for g in Gs], M_ref, lr=0.05, wd=0.3, cautious_wd=True,
                             neuron_state=V_ref, beta2=0.9, schedule=sched)
            torch.cuda.synchronize()
            assert nsb.muon_get_status() == 0
            for i in range(len(shapes)):
                assert torch.equal(sm.params[i], W_ref[i]), (step, i)
                assert torch.equal(sm.momentum[i], M_ref[i]), (step, i)
                assert torch.equal(sm.neuron_state[i], V_ref[i]), (step, i)
    finally:
        dist.destroy_process_group()
