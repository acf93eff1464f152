"""The sharded Muon step's host logic on CPU: ownership, and two gloo ranks.

The step over a data-parallel group must equal the single-process step on the
group-averaged gradients (each matrix's update is independent of the
others), on every rank.  The local step here is the oracle's fp64 Muon step
run on CPU tensors, so the comparison with a single process running the same
oracle on the averaged gradients is exact.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp
from hypothesis import given, settings, strategies as st

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from newton_schulz_12_b200.sharded import ns_flops, plan_ownership  # noqa: E402
from oracle import muon as oracle  # noqa: E402

SHAPES = [(16, 24), (24, 16), (32, 32), (8, 40), (40, 8), (12, 12)] * 2 + [(20, 20)]
HYPER = dict(beta=0.95, nesterov=True, lr=0.05, wd=0.01, steps=5)


def oracle_local_step(params, grads, bufs, beta, nesterov, lr, wd, steps):
    for W, G, M in zip(params, grads, bufs):
        Wn, Mn, _ = oracle.muon_step(W.double().numpy(), G.double().numpy(), M.double().numpy(),
                                     beta=beta, nesterov=nesterov, lr=lr, wd=wd, steps=steps)
        W.copy_(torch.from_numpy(Wn).float())
        M.copy_(torch.from_numpy(Mn).float())


def oracle_local_step_ex(params, grads, bufs, beta, nesterov, lr, wd, steps, cautious_wd=False,
                         neuron_state=None, beta2=0.95, schedule=None):
    """The oracle's step with the refinements; the NorMuon state updated in place."""
    for k, (W, G, M) in enumerate(zip(params, grads, bufs)):
        v = None if neuron_state is None else neuron_state[k].double().numpy()
        Wn, Mn, _, vn = oracle.muon_step_ex(W.double().numpy(), G.double().numpy(), M.double().numpy(),
                                            beta=beta, nesterov=nesterov, lr=lr, wd=wd, steps=steps,
                                            cautious=cautious_wd, neuron_state=v, beta2=beta2,
                                            schedule=schedule)
        W.copy_(torch.from_numpy(Wn).float())
        M.copy_(torch.from_numpy(Mn).float())
        if neuron_state is not None:
            neuron_state[k].copy_(torch.from_numpy(vn).float())


def initial_w(i, shape):
    g = torch.Generator().manual_seed(2000 + i)
    return torch.randn(shape, generator=g) * 0.02


def rank_grad(i, shape, rank, step):
    g = torch.Generator().manual_seed(1000 + 100 * step + 10 * rank + i)
    return torch.randn(shape, generator=g) * 0.01


# ----------------------------------------------------------------- ownership
def test_flops_match_the_oracle_count():
    for r, c in [(768, 768), (768, 3072), (3072, 768), (5, 77)]:
        assert ns_flops((r, c)) == oracle.ns_flops(r, c)


@pytest.mark.parametrize("world,buckets", [(1, 1), (2, 2), (3, 1), (8, 2), (5, 4)])
def test_every_matrix_has_one_owner_and_buckets_are_balanced(world, buckets):
    shapes = [(768, 768)] * 4 + [(768, 3072), (3072, 768)]
    shapes = shapes * 12  # the GPT-2-small hidden set in layer order
    owner, ranges = plan_ownership(shapes, world, buckets)
    assert len(owner) == len(shapes) and all(0 <= r < world for r in owner)
    assert ranges[0][0] == 0 and ranges[-1][1] == len(shapes)
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    for lo, hi in ranges:
        load = [0] * world
        for i in range(lo, hi):
            load[owner[i]] += ns_flops(shapes[i])
        biggest = max(ns_flops(shapes[i]) for i in range(lo, hi))
        # greedy longest-first: no rank exceeds the mean by more than one item
        assert max(load) <= sum(load) / world + biggest
    assert plan_ownership(shapes, world, buckets) == (owner, ranges)  # deterministic


@settings(max_examples=200, deadline=None)
@given(shapes=st.lists(st.tuples(st.integers(1, 4096), st.integers(1, 4096)), min_size=0, max_size=40),
       world=st.integers(1, 9), buckets=st.integers(1, 6), steps=st.integers(0, 7))
def test_ownership_properties(shapes, world, buckets, steps):
    """Any shapes, group size and bucket count: one owner per matrix, buckets
    tile the list in order, every bucket within one item of its mean load."""
    owner, ranges = plan_ownership(shapes, world, buckets, steps)
    assert len(owner) == len(shapes) and all(0 <= r < world for r in owner)
    if not shapes:
        assert ranges == [(0, 0)] or ranges == []
        return
    assert ranges[0][0] == 0 and ranges[-1][1] == len(shapes)
    assert all(a[1] == b[0] and a[0] < a[1] for a, b in zip(ranges, ranges[1:]))
    assert len(ranges) == min(buckets, len(shapes))
    for lo, hi in ranges:
        load = [0] * world
        for i in range(lo, hi):
            load[owner[i]] += ns_flops(shapes[i], steps)
        biggest = max(ns_flops(shapes[i], steps) for i in range(lo, hi))
        assert max(load) <= sum(load) / world + biggest
    assert plan_ownership(shapes, world, buckets, steps) == (owner, ranges)


def test_longest_first_on_a_small_case():
    """Squares of 64, 56, 48, 40 (costs proportional to 262144, 175616, 110592,
    64000) on two ranks, listed out of order: 64 -> r0, 56 -> r1, 48 -> r1
    (175616 < 262144), 40 -> r0 (262144 < 286208)."""
    shapes = [(48, 48), (64, 64), (40, 40), (56, 56)]
    owner, _ = plan_ownership(shapes, 2, 1)
    assert owner == [1, 0, 0, 1]


def test_arguments_are_checked_before_any_allocation():
    from newton_schulz_12_b200.sharded import ShardedMuon
    with pytest.raises(ValueError, match="device='cuda'"):
        ShardedMuon([(8, 8)])  # the CUDA step on a CPU device
    with pytest.raises(ValueError, match="device='cuda'"):
        ShardedMuon([(8, 8)], device="cuda", grad_dtype=torch.float32)
    with pytest.raises(ValueError, match="two positive sizes"):
        ShardedMuon([(8, 0)], local_step=oracle_local_step)


def test_no_matrices_is_a_no_op():
    from newton_schulz_12_b200.sharded import ShardedMuon
    sm = ShardedMuon([], local_step=oracle_local_step)
    sm.step()
    assert sm.params == [] and sm.bucket_ranges == []


def test_learning_rate_schedule_per_step():
    """step(lr=, wd=) changes the values the local step receives from then on."""
    from newton_schulz_12_b200.sharded import ShardedMuon
    seen = []

    def record(params, grads, bufs, beta, nesterov, lr, wd, steps):
        seen.append((lr, wd))

    sm = ShardedMuon(SHAPES[:3], buckets=1, grad_dtype=torch.float32, local_step=record, **HYPER)
    sm.step()
    sm.step(lr=0.02)
    sm.step(wd=0.5)
    sm.step()
    assert seen == [(0.05, 0.01), (0.02, 0.01), (0.02, 0.5), (0.02, 0.5)]


def test_single_rank_step_equals_oracle_step():
    from newton_schulz_12_b200.sharded import ShardedMuon
    sm = ShardedMuon(SHAPES, buckets=3, grad_dtype=torch.float32, local_step=oracle_local_step,
                     **HYPER)
    W0 = [initial_w(i, s) for i, s in enumerate(SHAPES)]
    for i, w in enumerate(W0):
        sm.params[i].copy_(w)
        sm.grads[i].copy_(rank_grad(i, SHAPES[i], 0, 0))
    sm.step()
    for i, s in enumerate(SHAPES):
        Wn, _, _ = oracle.muon_step(W0[i].double().numpy(), rank_grad(i, s, 0, 0).double().numpy(),
                                    np.zeros(s), **HYPER)
        np.testing.assert_array_equal(sm.params[i].numpy(), Wn.astype(np.float32))


# ------------------------------------------------------------ two gloo ranks
def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, buckets, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from newton_schulz_12_b200.sharded import ShardedMuon
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        sm = ShardedMuon(SHAPES, buckets=buckets, grad_dtype=torch.float32,
                         local_step=oracle_local_step, **HYPER)
        for i, s in enumerate(SHAPES):
            sm.params[i].copy_(initial_w(i, s))
        for step in range(2):
            for i, s in enumerate(SHAPES):
                sm.grads[i].copy_(rank_grad(i, s, rank, step))
            sm.step()
        out.put((rank, [p.clone().numpy() for p in sm.params],
                 {i: m.clone().numpy() for i, m in enumerate(sm.momentum) if m is not None}))
    finally:
        dist.destroy_process_group()


def _run_ranks(world, target, *args):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=target, args=(r, world, port) + args + (q,)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return res


def _run_two_ranks(buckets):
    return _run_ranks(2, _worker, buckets)


def _single_process_reference():
    W = [initial_w(i, s).double().numpy() for i, s in enumerate(SHAPES)]
    M = [np.zeros(s) for s in SHAPES]
    for step in range(2):
        for i, s in enumerate(SHAPES):
            # the group mean, in the fp32 order the ranks use: (g0 + g1) / 2
            g = (rank_grad(i, s, 0, step) + rank_grad(i, s, 1, step)) / 2
            Wn, Mn, _ = oracle.muon_step(W[i], g.double().numpy(), M[i], **HYPER)
            W[i] = Wn.astype(np.float32).astype(np.float64)
            M[i] = Mn.astype(np.float32).astype(np.float64)
    return W, M


@pytest.mark.parametrize("buckets", [1, 3])
def test_two_gloo_ranks_equal_the_single_process_step(buckets):
    res = _run_two_ranks(buckets)
    W_ref, M_ref = _single_process_reference()
    owner, _ = plan_ownership(SHAPES, 2, buckets)
    for rank, params, moms in res:
        for i in range(len(SHAPES)):
            np.testing.assert_array_equal(params[i], W_ref[i].astype(np.float32),
                                          err_msg=f"rank {rank} matrix {i}")
        # momentum lives with the owner only
        assert sorted(moms) == [i for i in range(len(SHAPES)) if owner[i] == rank]
        for i, m in moms.items():
            np.testing.assert_array_equal(m, M_ref[i].astype(np.float32))


# ------------------------------------- two gloo ranks with the refinements on
REFINE = dict(cautious_wd=True, normuon=True, beta2=0.9,
              schedule=[(3.4445, -4.7750, 2.0315)] * 3 + [(15 / 8, -10 / 8, 3 / 8), (1.5, -0.5, 0.0)])
HYPER_R = dict(HYPER, wd=0.3)
del HYPER_R["steps"]


def _worker_refined(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from newton_schulz_12_b200.sharded import ShardedMuon
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        sm = ShardedMuon(SHAPES, buckets=2, grad_dtype=torch.float32,
                         local_step=oracle_local_step_ex, **HYPER_R, **REFINE)
        for i, s in enumerate(SHAPES):
            sm.params[i].copy_(initial_w(i, s))
        for step in range(2):
            for i, s in enumerate(SHAPES):
                sm.grads[i].copy_(rank_grad(i, s, rank, step))
            sm.step()
        out.put((rank, [p.clone().numpy() for p in sm.params],
                 {i: v.clone().numpy() for i, v in enumerate(sm.neuron_state) if v is not None}))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_with_refinements_equal_the_single_process_step():
    """Cautious decay, NorMuon's state (kept by the owner) and a per-step
    schedule: the group step equals the single-process step_ex on the
    averaged gradients, state included."""
    res = _run_ranks(2, _worker_refined)
    W = [initial_w(i, s).double().numpy() for i, s in enumerate(SHAPES)]
    M = [np.zeros(s) for s in SHAPES]
    V = [np.zeros(s[0]) for s in SHAPES]
    for step in range(2):
        for i, s in enumerate(SHAPES):
            g = (rank_grad(i, s, 0, step) + rank_grad(i, s, 1, step)) / 2
            Wn, Mn, _, vn = oracle.muon_step_ex(W[i], g.double().numpy(), M[i], **HYPER_R,
                                                cautious=True, neuron_state=V[i], beta2=0.9,
                                                schedule=REFINE["schedule"])
            W[i] = Wn.astype(np.float32).astype(np.float64)
            M[i] = Mn.astype(np.float32).astype(np.float64)
            V[i] = vn.astype(np.float32).astype(np.float64)
    owner, _ = plan_ownership(SHAPES, 2, 2, steps=5)
    for rank, params, states in res:
        for i in range(len(SHAPES)):
            np.testing.assert_array_equal(params[i], W[i].astype(np.float32),
                                          err_msg=f"rank {rank} matrix {i}")
        assert sorted(states) == [i for i in range(len(SHAPES)) if owner[i] == rank]
        for i, v in states.items():
            np.testing.assert_array_equal(v, V[i].astype(np.float32))


def test_refinement_options_reach_the_local_step():
    from newton_schulz_12_b200.sharded import ShardedMuon
    seen = []

    def record(params, grads, bufs, beta, nesterov, lr, wd, steps, **kw):
        seen.append((steps, kw))

    ShardedMuon(SHAPES[:2], buckets=1, grad_dtype=torch.float32, local_step=record, **HYPER).step()
    assert seen == [(5, {})]  # nothing on: the plain call
    seen.clear()
    sm = ShardedMuon(SHAPES[:2], buckets=1, grad_dtype=torch.float32, local_step=record,
                     **HYPER_R, **REFINE)
    sm.step()
    steps, kw = seen[0]
    assert steps == 5 and kw["cautious_wd"] and kw["beta2"] == 0.9
    assert kw["schedule"] == [tuple(float(v) for v in t) for t in REFINE["schedule"]]
    assert [tuple(v.shape) for v in kw["neuron_state"]] == [(16,), (24,)]


# ------------------------------------------------------- checkpoint / resume
def _worker_ckpt(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from newton_schulz_12_b200.sharded import ShardedMuon
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        sm = ShardedMuon(SHAPES, buckets=2, grad_dtype=torch.float32,
                         local_step=oracle_local_step_ex, **HYPER_R, **REFINE)
        for i, s in enumerate(SHAPES):
            sm.params[i].copy_(initial_w(i, s))
        for step in range(2):
            for i, s in enumerate(SHAPES):
                sm.grads[i].copy_(rank_grad(i, s, rank, step))
            sm.step(lr=0.04 if step == 1 else None)
        st = sm.state_dict()  # tensors leave the process as arrays
        st = dict(st, momentum={i: t.numpy() for i, t in st["momentum"].items()},
                  neuron_state={i: t.numpy() for i, t in st["neuron_state"].items()})
        out.put((rank, [p.clone().numpy() for p in sm.params], st))
    finally:
        dist.destroy_process_group()


def test_checkpoint_from_two_ranks_resumes_on_one():
    """Two gloo ranks take two steps (the second with a new lr) and save;
    their states, merged, resume on a single rank: the third step equals
    three uninterrupted single-process steps on the averaged gradients, bit
    for bit (weights, momentum, NorMuon state)."""
    from newton_schulz_12_b200.sharded import ShardedMuon
    res = _run_ranks(2, _worker_ckpt)
    merged = {"momentum": {}, "neuron_state": {}}
    for _, _, st in res:
        merged["hyper"], merged["shapes"] = st["hyper"], st["shapes"]
        merged["momentum"].update({i: torch.from_numpy(a) for i, a in st["momentum"].items()})
        merged["neuron_state"].update({i: torch.from_numpy(a) for i, a in st["neuron_state"].items()})
    assert sorted(merged["momentum"]) == list(range(len(SHAPES)))
    sm = ShardedMuon(SHAPES, buckets=3, grad_dtype=torch.float32, local_step=oracle_local_step_ex,
                     **HYPER_R, **REFINE)
    sm.load_state_dict(merged)
    assert sm.hyper[2] == 0.04
    for i, p in enumerate(res[0][1]):
        sm.params[i].copy_(torch.from_numpy(p))
    for i, s in enumerate(SHAPES):
        sm.grads[i].copy_((rank_grad(i, s, 0, 2) + rank_grad(i, s, 1, 2)) / 2)
    sm.step()
    W = [initial_w(i, s).double().numpy() for i, s in enumerate(SHAPES)]
    M = [np.zeros(s) for s in SHAPES]
    V = [np.zeros(s[0]) for s in SHAPES]
    for step in range(3):
        hyper = dict(HYPER_R, lr=0.05 if step == 0 else 0.04)
        for i, s in enumerate(SHAPES):
            g = (rank_grad(i, s, 0, step) + rank_grad(i, s, 1, step)) / 2
            Wn, Mn, _, vn = oracle.muon_step_ex(W[i], g.double().numpy(), M[i], **hyper, cautious=True,
                                                neuron_state=V[i], beta2=0.9,
                                                schedule=REFINE["schedule"])
            W[i] = Wn.astype(np.float32).astype(np.float64)
            M[i] = Mn.astype(np.float32).astype(np.float64)
            V[i] = vn.astype(np.float32).astype(np.float64)
    for i in range(len(SHAPES)):
        np.testing.assert_array_equal(sm.params[i].numpy(), W[i].astype(np.float32))
        np.testing.assert_array_equal(sm.momentum[i].numpy(), M[i].astype(np.float32))
        np.testing.assert_array_equal(sm.neuron_state[i].numpy(), V[i].astype(np.float32))


def test_load_state_dict_checks():
    from newton_schulz_12_b200.sharded import ShardedMuon
    sm = ShardedMuon(SHAPES[:3], buckets=1, grad_dtype=torch.float32, local_step=oracle_local_step,
                     **HYPER)
    st = sm.state_dict()
    assert sorted(st["momentum"]) == [0, 1, 2] and "neuron_state" not in st
    with pytest.raises(ValueError, match="shapes"):
        ShardedMuon(SHAPES[:2], buckets=1, grad_dtype=torch.float32,
                    local_step=oracle_local_step, **HYPER).load_state_dict(st)
    partial = dict(st, momentum={0: st["momentum"][0]})
    with pytest.raises(ValueError, match="missing"):
        sm.load_state_dict(partial)
    refined = ShardedMuon(SHAPES[:3], buckets=1, grad_dtype=torch.float32,
                          local_step=oracle_local_step_ex, normuon=True, **HYPER)
    with pytest.raises(ValueError, match="NorMuon"):
        refined.load_state_dict(st)


# ------------------------------------------- three ranks, one idle in a bucket
SHAPES3 = [(16, 24), (24, 16), (32, 32), (8, 40)]


def exact_grad(i, shape, rank):
    """Integers times 2^-14: their three-rank sums are exact in any order."""
    g = torch.Generator().manual_seed(4000 + 10 * rank + i)
    return torch.round(torch.randn(shape, generator=g) * 160) / 2 ** 14


def _worker3(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from newton_schulz_12_b200.sharded import ShardedMuon
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        sm = ShardedMuon(SHAPES3, buckets=2, grad_dtype=torch.float32,
                         local_step=oracle_local_step, **HYPER)
        for i, s in enumerate(SHAPES3):
            sm.params[i].copy_(initial_w(i, s))
            sm.grads[i].copy_(exact_grad(i, s, rank))
        sm.step()
        out.put((rank, [p.clone().numpy() for p in sm.params], sm.owner))
    finally:
        dist.destroy_process_group()


def test_three_ranks_with_an_idle_rank_in_a_bucket():
    owner, ranges = plan_ownership(SHAPES3, 3, 2)
    assert ranges == [(0, 2), (2, 4)]
    assert 2 not in owner[0:2]  # rank 2 owns nothing in bucket 0 yet joins its collectives
    res = _run_ranks(3, _worker3)
    for rank, params, own in res:
        assert own == owner
        for i, s in enumerate(SHAPES3):
            g = (exact_grad(i, s, 0) + exact_grad(i, s, 1) + exact_grad(i, s, 2)) / 3
            Wn, _, _ = oracle.muon_step(initial_w(i, s).double().numpy(), g.double().numpy(),
                                        np.zeros(s), **HYPER)
            np.testing.assert_array_equal(params[i], Wn.astype(np.float32),
                                          err_msg=f"rank {rank} matrix {i}")


# ------------------------------------------- bf16 gradients on a backend without reduce-scatter
def _worker_bf16(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    from newton_schulz_12_b200.sharded import ShardedMuon
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        seen = {}

        def record(params, grads, bufs, beta, nesterov, lr, wd, steps):
            for g in grads:
                seen[g.data_ptr()] = g.clone()

        sm = ShardedMuon(SHAPES, buckets=2, grad_dtype=torch.bfloat16, local_step=record, **HYPER)
        for i, s in enumerate(SHAPES):
            sm.grads[i].copy_(rank_grad(i, s, rank, 0) * 37.0)  # bf16 values of mixed exponents
        ptr = {i: sm.grads[i].data_ptr() for i in range(len(SHAPES))}
        sm.step()
        out.put((rank, {i: seen[ptr[i]].float().numpy() for i in range(len(SHAPES)) if ptr[i] in seen}))
    finally:
        dist.destroy_process_group()


def test_bf16_gradients_are_averaged_in_fp32():
    """Without reduce-scatter (gloo) the owner receives the fp32 mean of the
    bf16 gradients rounded once to bf16 -- not a bf16 sum divided afterwards."""
    res = _run_ranks(2, _worker_bf16)
    owner, _ = plan_ownership(SHAPES, 2, 2)
    for rank, got in res:
        assert sorted(got) == [i for i in range(len(SHAPES)) if owner[i] == rank]
        for i, g in got.items():
            a = (rank_grad(i, SHAPES[i], 0, 0) * 37.0).to(torch.bfloat16).float()
            b = (rank_grad(i, SHAPES[i], 1, 0) * 37.0).to(torch.bfloat16).float()
            want = ((a + b) / 2).to(torch.bfloat16).float().numpy()
            np.testing.assert_array_equal(g, want, err_msg=f"matrix {i}")
