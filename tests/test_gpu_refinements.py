"""Cautious weight decay, NorMuon's per-neuron rescale and per-step
coefficients in the full step on the GPU.

The pages name both refinements of the Muon update without formulas ("The
NanoGPT speedrun", paragraph "Reading guide"); the readings are those of
oracle/muon.py (cautious_mask, normuon_rescale) and include/muon.h.

* muon_apply_ex (the apply pass) bit for bit against the fp32 restatement,
  with cautious decay and with per-row factors;
* muon_step_ex end to end against the fp64 oracle on the GPU's own pre-step
  state: W' - W within relative Frobenius 3e-2 and every 32 x 32 block within
  4 x 3e-2; the momentum bit-exact; the NorMuon state v' over three steps so
  the state carries.

The state's bound follows from the update's.  Fed the same pre-step state,
GPU and oracle differ in v' only through r_i = mean_j O_ij^2.  If O's
whole-matrix relative error is d, then sum_i |dr_i| <= (2d + d^2) sum_i r_i
(expand |O_i|^2 - |O'_i|^2 and apply Cauchy-Schwarz), and the moving
average only shrinks that: the L1-relative error of v' is at most 2d + d^2.
Per row, with the 4 x 3e-2 a 32 x 32 block may carry as d, the same
expansion gives 2d + d^2 for that row.  The GPU sums the squares of O
rounded to bf16 (|O - hi| <= 2^-8 |hi|), each within a relative
2^-7 + 2^-14 of O's square, which adds at most that times (1 + d)^2 to
either bound.
"""
import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from blockcheck import assert_blocks
from newton_schulz_12_b200 import workloads
from oracle import muon as oracle
from oracle.fp32_ref import apply_f32, momentum_f32, update_scale_f32

pytestmark = pytest.mark.gpu

TOL = 3e-2
BF16_SQ = 2.0 ** -7 + 2.0 ** -14                  # relative error of a bf16 square
STATE_L1_TOL = 2 * TOL + TOL ** 2 + BF16_SQ * (1 + TOL) ** 2                  # whole vector, L1-relative
STATE_ROW_TOL = 2 * (4 * TOL) + (4 * TOL) ** 2 + BF16_SQ * (1 + 4 * TOL) ** 2  # each row


def rel_fro(got, ref):
    return float(np.linalg.norm(np.asarray(got, np.float64) - ref) / np.linalg.norm(ref))


# --------------------------------------------------------------- apply pass
APPLY_SHAPES = [(768, 3072), (3072, 768), (77, 5), (130, 68), (1, 40)]


@pytest.mark.parametrize("cautious", [False, True])
@pytest.mark.parametrize("rows_scaled", [False, True])
def test_apply_ex_bitwise(cautious, rows_scaled):
    W = [workloads.gaussian(s, 2e-2, seed=i).cuda() for i, s in enumerate(APPLY_SHAPES)]
    O = [workloads.gaussian(s, 1.0, seed=10 + i) for i, s in enumerate(APPLY_SHAPES)]
    for o in O:
        o.view(-1)[::7] = 0.0      # zeros: never decayed under the cautious mask
    F = [workloads.gaussian((s[0],), 0.5, seed=20 + i).abs() + 0.5 for i, s in enumerate(APPLY_SHAPES)]
    W0 = [w.cpu().numpy() for w in W]
    nsb.muon_apply_ex(W, [o.cuda() for o in O], lr=0.05, wd=3.0, cautious_wd=cautious,
                      row_scale=[f.cuda() for f in F] if rows_scaled else None)
    assert nsb.muon_get_status() == 0
    for i, (r, c) in enumerate(APPLY_SHAPES):
        ref = apply_f32(W0[i], O[i].numpy(), 0.05, 3.0, update_scale_f32(r, c), cautious=cautious,
                        row_scale=F[i].numpy() if rows_scaled else None)
        assert np.array_equal(W[i].cpu().numpy().view(np.uint32), ref.view(np.uint32)), (r, c)


# ------------------------------------------------------------- full step
class State:
    def __init__(self, shapes, normuon):
        self.shapes = shapes
        Ws, _ = workloads.muon_set(shapes, step=0)
        self.W = [w.cuda() for w in Ws]
        self.M = [torch.zeros(r, c, device="cuda") for r, c in shapes]
        self.V = [torch.zeros(r, device="cuda") for r, _ in shapes] if normuon else None


def check_step_ex(st, step, cautious, beta2=0.95, lr=0.05, wd=0.0, steps=5, check=None, schedule=None):
    _, Gs = workloads.muon_set(st.shapes, step=step)
    W0 = [w.cpu().numpy() for w in st.W]
    M0 = [m.cpu().numpy() for m in st.M]
    V0 = [v.cpu().numpy() for v in st.V] if st.V is not None else None
    nsb.muon_step_ex(st.W, [g.cuda() for g in Gs], st.M, lr=lr, wd=wd, steps=steps,
                     cautious_wd=cautious, neuron_state=st.V, beta2=beta2, schedule=schedule)
    if schedule is not None:  # the triples as the library received them (fp32)
        schedule = [tuple(float(np.float32(v)) for v in t) for t in schedule]
    assert nsb.muon_get_status() == 0
    for i in (range(len(st.shapes)) if check is None else check):
        g32 = Gs[i].float().numpy()
        nb32, _ = momentum_f32(g32, M0[i], 0.95, True)
        assert np.array_equal(st.M[i].cpu().numpy().view(np.uint32), nb32.view(np.uint32))
        Wn, _, _, vn = oracle.muon_step_ex(
            W0[i], g32, M0[i], beta=np.float32(0.95), lr=np.float32(lr), wd=np.float32(wd),
            steps=steps, cautious=cautious, neuron_state=None if V0 is None else V0[i],
            beta2=np.float32(beta2), schedule=schedule)
        dW_ref = Wn - W0[i]
        dW = st.W[i].cpu().numpy().astype(np.float64) - W0[i]
        err = rel_fro(dW, dW_ref)
        assert err <= TOL, f"matrix {i} {st.shapes[i]}: rel err {err:.3e}"
        assert_blocks(dW, dW_ref, 4 * TOL, f"matrix {i} {st.shapes[i]}")
        if V0 is not None:
            v = st.V[i].cpu().numpy().astype(np.float64)
            l1 = np.sum(np.abs(v - vn)) / np.sum(np.abs(vn))
            rel = np.abs(v - vn) / np.abs(vn)
            assert l1 <= STATE_L1_TOL, f"matrix {i}: state L1-relative error {l1:.3e}"
            assert rel.max() <= STATE_ROW_TOL, f"matrix {i}: state row error {rel.max():.3e}"


MIX = [(300, 1000), (1000, 300), (256, 256), (130, 68), (68, 130), (77, 5), (5, 77), (1, 40), (40, 1)]


def test_cautious_step_mixed_shapes():
    st = State(MIX, normuon=False)
    for step in range(2):
        check_step_ex(st, step, cautious=True, lr=0.05, wd=0.5)


def test_normuon_step_mixed_shapes_three_steps():
    st = State(MIX, normuon=True)
    for step in range(3):
        check_step_ex(st, step, cautious=False, wd=0.01)


def test_normuon_and_cautious_together():
    st = State(MIX[:5], normuon=True)
    for step in range(2):
        check_step_ex(st, step, cautious=True, beta2=0.9, wd=0.5)


@pytest.mark.parametrize("steps", [0, 1])
def test_normuon_few_steps(steps):
    """steps = 0: O is the normalised update itself (the scaled pair)."""
    st = State(MIX[:4], normuon=True)
    check_step_ex(st, 0, cautious=False, steps=steps)


# Per-step coefficients in the full step (the Polar Express reading: the
# pages print no coefficients, so the triples are the speedrun quintic, the
# flat quintic 15/8, -10/8, 3/8 and the classic cubic).
QUINTIC = (3.4445, -4.7750, 2.0315)
SCHEDULE = [QUINTIC, QUINTIC, (15 / 8, -10 / 8, 3 / 8), (1.5, -0.5, 0.0), (15 / 8, -10 / 8, 3 / 8)]


def test_schedule_step_mixed_shapes():
    """muon_step_ex with a schedule, alone and with both refinements, two
    steps, against the oracle step with the same triples."""
    st = State(MIX, normuon=False)
    for step in range(2):
        check_step_ex(st, step, cautious=False, wd=0.1, schedule=SCHEDULE)
    st = State(MIX[:5], normuon=True)
    for step in range(2):
        check_step_ex(st, step, cautious=True, wd=0.5, schedule=SCHEDULE[:4])


def test_default_schedule_is_muon_step():
    """The default triple at every step gives muon_step's bits (weights and momentum)."""
    shapes = MIX + workloads.gpt2_small_shapes()[:6]
    a, b = State(shapes, normuon=False), State(shapes, normuon=False)
    _, Gs = workloads.muon_set(shapes, step=0)
    nsb.muon_step(a.W, [g.cuda() for g in Gs], a.M, wd=0.1)
    nsb.muon_step_ex(b.W, [g.cuda() for g in Gs], b.M, wd=0.1, schedule=[QUINTIC] * 5)
    assert nsb.muon_get_status() == 0
    for i in range(len(shapes)):
        assert torch.equal(a.W[i], b.W[i]) and torch.equal(a.M[i], b.M[i]), shapes[i]


def test_gpt2_small_set_refinements():
    """The GPT-2-small hidden set (72 matrices) with both refinements, two
    steps, every matrix checked."""
    st = State(workloads.gpt2_small_shapes(), normuon=True)
    for step in range(2):
        check_step_ex(st, step, cautious=True, wd=0.1)


def test_no_options_is_muon_step():
    shapes = [(256, 768), (768, 256), (256, 256)]
    a, b = State(shapes, False), State(shapes, False)
    _, Gs = workloads.muon_set(shapes, step=0)
    nsb.muon_step(a.W, [g.cuda() for g in Gs], a.M, wd=0.1)
    nsb.muon_step_ex(b.W, [g.cuda() for g in Gs], b.M, wd=0.1)
    for x, y in zip(a.W, b.W):
        assert torch.equal(x, y)
