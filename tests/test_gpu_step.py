"""muon_step / muon_momentum / muon_apply (C ABI) against the oracle.

* momentum buffers: bit-exact against the fp32 restatement of the same order;
* apply: bit-exact against the fp32 restatement given the same update;
* the full step: the weight update W' - W within relative Frobenius 3e-2 of the
  fp64 oracle run on the GPU's own pre-step state (so no drift accumulates),
  and every 32 x 32 block of it within 4 x 3e-2 of the same block;
* the GPT-2-small hidden set (72 matrices, 768 wide) at full size, with
  Gaussian and with hard (log-uniform, spiked) gradient spectra;
* ten consecutive steps against the oracle run on its own state (no drift),
  and a non-finite gradient isolated to its own matrix.
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
BLOCK_TOL = 4 * TOL  # every 32 x 32 block of W' - W (tests/blockcheck.py)


def rel_fro(got, ref):
    return float(np.linalg.norm(np.asarray(got, np.float64) - ref) / np.linalg.norm(ref))


class State:
    def __init__(self, shapes, hard=False, w_seed=2000):
        self.shapes = shapes
        self.hard = hard
        Ws, _ = workloads.muon_set(shapes, step=0, w_seed=w_seed)
        self.W = [w.cuda() for w in Ws]
        self.M = [torch.zeros(r, c, device="cuda") for r, c in shapes]

    def grads(self, step):
        _, Gs = workloads.muon_set(self.shapes, step=step, hard=self.hard)
        return Gs


def check_step(st, step, beta=0.95, nesterov=True, lr=0.05, wd=0.0, steps=5, check=None):
    Gs = st.grads(step)
    W0 = [w.cpu().numpy() for w in st.W]
    M0 = [m.cpu().numpy() for m in st.M]
    nsb.muon_step(st.W, [g.cuda() for g in Gs], st.M, beta=beta, nesterov=nesterov, lr=lr, wd=wd,
                  steps=steps)
    assert nsb.muon_get_status() == 0
    idx = range(len(st.shapes)) if check is None else check
    worst = 0.0
    for i in idx:
        g32 = Gs[i].float().numpy()
        nb32, _ = momentum_f32(g32, M0[i], beta, nesterov)
        assert np.array_equal(st.M[i].cpu().numpy().view(np.uint32), nb32.view(np.uint32)), \
            f"momentum of matrix {i} not bit-exact"
        Wn, _, _ = oracle.muon_step(W0[i], g32, M0[i], beta=np.float32(beta), nesterov=nesterov,
                                    lr=np.float32(lr), wd=np.float32(wd), steps=steps)
        dW_ref = Wn - W0[i]
        dW = st.W[i].cpu().numpy().astype(np.float64) - W0[i]
        err = rel_fro(dW, dW_ref)
        worst = max(worst, err)
        assert err <= TOL, f"matrix {i} {st.shapes[i]}: rel err {err:.3e}"
        assert_blocks(dW, dW_ref, BLOCK_TOL, f"matrix {i} {st.shapes[i]}")
    return worst


def test_small_set_three_steps():
    shapes = workloads.gpt2_small_shapes(layers=2, width=256) + [(200, 328), (328, 200), (72, 72), (1, 40)]
    st = State(shapes)
    for step in range(3):
        check_step(st, step)


def test_weight_decay_and_plain_momentum():
    shapes = [(256, 256), (256, 1024), (1024, 256)]
    st = State(shapes)
    check_step(st, 0, wd=0.01)
    check_step(st, 1, nesterov=False, beta=0.9, lr=0.02, wd=0.1)


def test_zero_steps_applies_normalised_update():
    st = State([(300, 200), (128, 256)])
    check_step(st, 0, steps=0)


def test_gpt2_small_full_set():
    """All 72 hidden matrices of GPT-2 small, two steps, every matrix checked."""
    st = State(workloads.gpt2_small_shapes())
    for step in range(2):
        worst = check_step(st, step)
    assert worst < TOL


def test_gpt2_small_hard_spectra():
    st = State(workloads.gpt2_small_shapes(), hard=True)
    check_step(st, 0)


def test_scaled_set_full():
    """144-matrix 1024-wide set with wd 0.01, every matrix checked (all 144
    take the fused apply of the last launch)."""
    shapes = workloads.scaled_shapes()
    st = State(shapes)
    check_step(st, 0, wd=0.01)


# The last step's BX applies its result to W in the GEMM epilogue.  These
# shapes cover W with X's layout (wide, square), W = X^T (tall), ragged edges
# both ways, a one-row X, and W rows that are not 16-byte strided (cols % 4 !=
# 0: written as X_T and applied by the separate pass) -- the same shape group
# holding both kinds, and more shape groups than one launch takes.
APPLY_MIX = [(300, 1000), (1000, 300), (256, 256), (130, 68), (68, 130), (77, 5), (5, 77),
             (4, 12), (12, 4), (1, 40), (40, 1)]


def test_fused_apply_layouts_and_edges():
    st = State(APPLY_MIX)
    for step in range(2):
        check_step(st, step)


def test_fused_apply_weight_decay_dominant():
    """lr * wd = 0.2: the decay term dominates W' - W, so a missing or wrong
    decay in the fused epilogue breaks the tolerance."""
    st = State(APPLY_MIX)
    check_step(st, 0, lr=0.01, wd=20.0)


@pytest.mark.parametrize("steps", [1, 2])
def test_fused_apply_few_steps(steps):
    """With one step the fused launch is also the one that folds in 1 / ||u||."""
    st = State(APPLY_MIX[:5])
    check_step(st, 0, steps=steps)


def test_fused_apply_table_overflow():
    """168 matrices in one launch: the first 160 (wide and tall alternating)
    are applied in the epilogue, the rest written as X_T and applied by the
    separate pass."""
    st = State([(64, 192), (192, 64)] * 84)
    check_step(st, 0, wd=0.5)


def test_momentum_stage_bit_exact_and_sumsq():
    shapes = [(768, 768), (333, 77), (5, 3), (1, 1)]
    _, Gs = workloads.muon_set(shapes, step=0)
    M = [workloads.gaussian(s, 1e-2, seed=50 + i).cuda() for i, s in enumerate(shapes)]
    M0 = [m.cpu().numpy() for m in M]
    out = torch.zeros(len(shapes), device="cuda")
    nsb.muon_momentum([g.cuda() for g in Gs], M, beta=0.95, nesterov=True, sumsq_out=out)
    for i in range(len(shapes)):
        nb, u = momentum_f32(Gs[i].float().numpy(), M0[i], 0.95, True)
        assert np.array_equal(M[i].cpu().numpy().view(np.uint32), nb.view(np.uint32))
        ref = float(np.sum(u.astype(np.float64) ** 2))
        assert abs(float(out[i]) - ref) <= 1e-6 * ref


def test_apply_stage_bit_exact():
    shapes = [(768, 3072), (3072, 768), (77, 5)]
    W = [workloads.gaussian(s, 2e-2, seed=i).cuda() for i, s in enumerate(shapes)]
    O = [workloads.gaussian(s, 1.0, seed=10 + i).cuda() for i, s in enumerate(shapes)]
    W0 = [w.cpu().numpy() for w in W]
    nsb.muon_apply(W, O, lr=0.05, wd=0.01)
    for i, (r, c) in enumerate(shapes):
        ref = apply_f32(W0[i], O[i].cpu().numpy(), 0.05, 0.01, update_scale_f32(r, c))
        assert np.array_equal(W[i].cpu().numpy().view(np.uint32), ref.view(np.uint32))


def test_step_is_deterministic():
    shapes = [(768, 768), (768, 3072), (3072, 768)]
    outs = []
    for _ in range(2):
        st = State(shapes)
        nsb.muon_step(st.W, [g.cuda() for g in st.grads(0)], st.M)
        outs.append([w.cpu().numpy() for w in st.W])
    for a, b in zip(*outs):
        assert np.array_equal(a, b)


def test_empty_count_is_noop():
    nsb.muon_step([], [], [])
    assert nsb.muon_get_status() == 0


@pytest.mark.parametrize("bad", [float("nan"), float("inf")])
def test_non_finite_gradient_leaves_the_other_matrices_unchanged(bad):
    """A NaN or inf in one matrix's gradient changes no bit of any other
    matrix's weights or momentum (same shape group and other groups)."""
    shapes = [(256, 256), (256, 1024), (1024, 256), (256, 256), (256, 1024)]
    Ws, Gs = workloads.muon_set(shapes, step=0)
    runs = []
    for poison in (False, True):
        W = [w.cuda() for w in Ws]
        M = [torch.zeros(s, device="cuda") for s in shapes]
        G = [g.clone().cuda() for g in Gs]
        if poison:
            G[1][3, 9] = bad
        nsb.muon_step(W, G, M, wd=0.01)
        torch.cuda.synchronize()
        runs.append(([w.cpu() for w in W], [m.cpu() for m in M]))
    (Wc, Mc), (Wp, Mp) = runs
    for i in (0, 2, 3, 4):
        assert torch.equal(Wc[i], Wp[i]) and torch.equal(Mc[i], Mp[i]), i


def test_ten_steps_track_the_oracle():
    """Ten consecutive steps from the same start, the GPU on its own state and
    the fp64 oracle on its own (momentum and weights never re-synchronised):
    the total change of W stays within 3e-2 of the oracle's, relative in
    Frobenius norm, for every matrix, and within 4 x 3e-2 on every 32 x 32
    block -- no error builds up in the momentum or the weights over steps."""
    shapes = workloads.gpt2_small_shapes(layers=1, width=256) + [(130, 68)]
    Ws, _ = workloads.muon_set(shapes, step=0)
    W = [w.cuda() for w in Ws]
    M = [torch.zeros(s, device="cuda") for s in shapes]
    Wo = [w.double().numpy() for w in Ws]
    Mo = [np.zeros(s) for s in shapes]
    for step in range(10):
        _, Gs = workloads.muon_set(shapes, step=step)
        nsb.muon_step(W, [g.cuda() for g in Gs], M, wd=0.01)
        for i in range(len(shapes)):
            Wo[i], Mo[i], _ = oracle.muon_step(Wo[i], Gs[i].double().numpy(), Mo[i], beta=np.float32(0.95),
                                               lr=np.float32(0.05), wd=np.float32(0.01))
    assert nsb.muon_get_status() == 0
    for i in range(len(shapes)):
        dW_ref = Wo[i] - Ws[i].double().numpy()
        dW = W[i].double().cpu().numpy() - Ws[i].double().numpy()
        assert rel_fro(dW, dW_ref) <= TOL, (i, shapes[i], rel_fro(dW, dW_ref))
        assert_blocks(dW, dW_ref, BLOCK_TOL, f"matrix {i} after ten steps")
