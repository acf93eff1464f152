"""A Muon step recorded in a CUDA graph and replayed (MuonStepPlan.capture /
replay) must give exactly what the same number of direct calls gives: the
library's launches are capture-safe once the stream's workspace exists, and
every kernel is deterministic, so the weights and momentum agree bit for bit
after several steps."""
import pytest
import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import workloads

pytestmark = pytest.mark.gpu


def _set(shapes):
    Ws, Gs = workloads.muon_set(shapes, step=0)
    return ([w.cuda() for w in Ws], [g.cuda() for g in Gs],
            [torch.zeros(w.shape, device="cuda") for w in Ws])


@pytest.mark.parametrize("shapes", [workloads.gpt2_small_shapes(layers=2),
                                    [(300, 1000), (1000, 300), (77, 5), (256, 256)]])
def test_graph_replay_equals_direct_calls(shapes):
    Wa, Ga, Ma = _set(shapes)
    Wb, Gb, Mb = [w.clone() for w in Wa], [g.clone() for g in Ga], [m.clone() for m in Ma]
    plan_a = nsb.MuonStepPlan(Wa, Ga, Ma, wd=0.01)
    plan_b = nsb.MuonStepPlan(Wb, Gb, Mb, wd=0.01)
    plan_a.capture()          # one step (the warm call; the captured step is only recorded)
    for _ in range(4):
        plan_a.replay()       # four more
    for _ in range(5):
        plan_b()
    torch.cuda.synchronize()
    assert nsb.muon_get_status() == 0
    for x, y in zip(Wa + Ma, Wb + Mb):
        assert torch.equal(x, y)


@pytest.mark.parametrize("m,n,batch", [(256, 256, 200), (130, 68, 3), (768, 3072, 2)])
def test_ns_plan_and_its_replay_equal_direct_calls(m, n, batch):
    """MuonNsPlan: a call equals muon_ns_orthogonalize; capture (one call) plus
    two replays equal three direct calls, bit for bit."""
    xs = [workloads.gaussian((m, n), 1.0, seed=40 + i, dtype=torch.bfloat16).cuda() for i in range(batch)]
    a = [x.clone() for x in xs]
    b = [x.clone() for x in xs]
    c = [x.clone() for x in xs]
    nsb.MuonNsPlan(a)()
    nsb.muon_ns_orthogonalize(b)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
    plan = nsb.MuonNsPlan(c)
    plan.capture()
    for _ in range(2):
        plan.replay()
    for _ in range(2):
        nsb.muon_ns_orthogonalize(b)
    torch.cuda.synchronize()
    assert nsb.muon_get_status() == 0
    assert all(torch.equal(x, y) for x, y in zip(c, b))


def test_refined_plan_replay_equals_muon_step_ex():
    """MuonStepPlan with the refinements (cautious decay, NorMuon state, a
    per-step schedule) calls muon_step_ex; recorded and replayed it gives the
    bits of direct muon_step_ex calls, weights, momentum and state."""
    shapes = workloads.gpt2_small_shapes(layers=1) + [(130, 68), (77, 5)]
    sched = [(3.4445, -4.7750, 2.0315)] * 4 + [(1.5, -0.5, 0.0)]
    Wa, Ga, Ma = _set(shapes)
    Wb, Gb, Mb = [w.clone() for w in Wa], [g.clone() for g in Ga], [m.clone() for m in Ma]
    Va = [torch.zeros(w.shape[0], device="cuda") for w in Wa]
    Vb = [v.clone() for v in Va]
    plan = nsb.MuonStepPlan(Wa, Ga, Ma, wd=0.2, cautious_wd=True, neuron_state=Va, beta2=0.9,
                            schedule=sched)
    plan.capture()
    for _ in range(2):
        plan.replay()
    for _ in range(3):
        nsb.muon_step_ex(Wb, Gb, Mb, wd=0.2, cautious_wd=True, neuron_state=Vb, beta2=0.9,
                         schedule=sched)
    torch.cuda.synchronize()
    assert nsb.muon_get_status() == 0
    for x, y in zip(Wa + Ma + Va, Wb + Mb + Vb):
        assert torch.equal(x, y)
    with pytest.raises(ValueError, match="schedule"):
        plan.update(steps=3)
