"""Muon over a data-parallel group: one process per GPU, torch.distributed.

Every rank holds the full set of hidden matrices W.  A step over the group is
the single-GPU step applied to the group-averaged gradients, with the work
split by matrix ("The NanoGPT speedrun", record #3: the Newton-Schulz
orthogonalisation of one matrix is independent of every other):

1. gradients are averaged and delivered to their owner only -- one
   reduce-scatter per bucket over a flat buffer laid out by owner;
2. each owner runs the Muon step (momentum, Newton-Schulz, apply) on the
   matrices it owns and keeps their momentum buffers;
3. the updated weights are all-gathered in place, so that every rank again
   holds the full set.

Bucket b's all-gather is issued asynchronously right after its local step,
so it runs on the communication stream while bucket b+1 is orthogonalised.

Ownership: the matrices are split into ``buckets`` contiguous runs in the
caller's order; inside a bucket each matrix, longest first by Newton-Schulz
FLOPs T(4 m^2 n + 2 m^3) (m <= n; ties by index), goes to the least-loaded
rank (ties to the lower rank), so every bucket's all-gather is balanced too.

Storage: per bucket one flat fp32 W buffer and one flat gradient buffer of
``world`` equal slots, slot r holding the matrices rank r owns (each start
padded to 64 elements, 16-byte aligned as the C ABI requires).  ``params``
and ``grads`` are views into them: the caller writes its gradients into
``grads`` and reads the weights from ``params``.
"""
from __future__ import annotations

import torch

_ALIGN = 64  # elements; every matrix view starts 256-byte aligned


def ns_flops(shape, steps=5):
    """Nominal Newton-Schulz FLOPs of one (r x c) matrix: T (4 m^2 n + 2 m^3), m <= n."""
    m, n = sorted((int(shape[0]), int(shape[1])))
    return steps * (4 * m * m * n + 2 * m ** 3)


def plan_ownership(shapes, world, buckets=2, steps=5):
    """Owner rank of every matrix and the [begin, end) index range of every bucket."""
    if world < 1:
        raise ValueError("world must be >= 1")
    k = len(shapes)
    nb = max(1, min(int(buckets), k)) if k else 0
    bounds = [round(b * k / nb) for b in range(nb + 1)] if nb else [0]
    owner = [0] * k
    for b in range(nb):
        load = [0] * world
        idx = range(bounds[b], bounds[b + 1])
        for i in sorted(idx, key=lambda i: (-ns_flops(shapes[i], steps), i)):
            r = min(range(world), key=lambda q: (load[q], q))
            owner[i] = r
            load[r] += ns_flops(shapes[i], steps)
    return owner, [(bounds[b], bounds[b + 1]) for b in range(nb)]


def _round_up(x, a):
    return (x + a - 1) // a * a


class ShardedMuon:
    """Muon step over the ranks of ``group`` (the default group when None).

    ``local_step(params, grads, momentum_bufs, beta, nesterov, lr, wd, steps)``
    updates the owned matrices in place; by default it is this package's
    ``muon_step`` (bf16 gradients on the CUDA device), prepared once per
    bucket.  Without an initialised process group the object runs as a
    single rank.

    The refinements of ``muon_step_ex`` ("The NanoGPT speedrun", paragraph
    "Reading guide"): ``cautious_wd``, ``normuon`` (NorMuon's per-neuron
    state, one fp32 vector per owned matrix in ``neuron_state``, kept by the
    owner like the momentum; ``beta2``) and ``schedule`` (one (a, b, c) per
    Newton-Schulz step; it sets ``steps``).  With any of them on, a custom
    ``local_step`` also receives the keywords ``cautious_wd``,
    ``neuron_state``, ``beta2`` and ``schedule``.
    """

    def __init__(self, shapes, *, device=None, group=None, buckets=2, beta=0.95, nesterov=True,
                 lr=0.05, wd=0.0, steps=5, grad_dtype=torch.bfloat16, local_step=None,
                 cautious_wd=False, normuon=False, beta2=0.95, schedule=None):
        import torch.distributed as dist
        for i, shp in enumerate(shapes):
            if len(shp) != 2 or int(shp[0]) < 1 or int(shp[1]) < 1:
                raise ValueError(f"shape {i} must be two positive sizes, got {tuple(shp)}")
        dev = torch.device(device) if device is not None else torch.device("cpu")
        if local_step is None and (dev.type != "cuda" or grad_dtype != torch.bfloat16):
            raise ValueError("the library's muon_step needs device='cuda' and bf16 gradients; "
                             "pass local_step for anything else")
        self.dist = dist if dist.is_available() and dist.is_initialized() else None
        self.group = group
        self.world = self.dist.get_world_size(group) if self.dist else 1
        self.rank = self.dist.get_rank(group) if self.dist else 0
        self.shapes = [(int(r), int(c)) for r, c in shapes]
        if schedule is not None:
            schedule = [tuple(float(v) for v in t) for t in schedule]
            if any(len(t) != 3 for t in schedule):
                raise ValueError("schedule must be a sequence of (a, b, c) triples")
            steps = len(schedule)
        self.options = None
        if cautious_wd or normuon or schedule is not None:
            self.options = dict(cautious_wd=bool(cautious_wd), beta2=float(beta2), schedule=schedule)
        self.hyper = (float(beta), bool(nesterov), float(lr), float(wd), int(steps))
        self.device = dev
        self.owner, self.bucket_ranges = plan_ownership(self.shapes, self.world, buckets, steps)
        self._nccl = bool(self.dist) and self.dist.get_backend(group) == "nccl"

        self.params = [None] * len(self.shapes)
        self.grads = [None] * len(self.shapes)
        self.momentum = [None] * len(self.shapes)
        self.neuron_state = [None] * len(self.shapes)
        self._buckets = []
        for lo, hi in self.bucket_ranges:
            offs, used = {}, [0] * self.world
            for i in range(lo, hi):
                r = self.owner[i]
                offs[i] = used[r]
                used[r] = _round_up(used[r] + self.shapes[i][0] * self.shapes[i][1], _ALIGN)
            slot = max(max(used), _ALIGN)
            W = torch.zeros(self.world * slot, dtype=torch.float32, device=self.device)
            G = torch.zeros(self.world * slot, dtype=grad_dtype, device=self.device)
            owned = []
            for i in range(lo, hi):
                r, (rows, cols) = self.owner[i], self.shapes[i]
                a = r * slot + offs[i]
                self.params[i] = W[a:a + rows * cols].view(rows, cols)
                self.grads[i] = G[a:a + rows * cols].view(rows, cols)
                if r == self.rank:
                    self.momentum[i] = torch.zeros(rows, cols, dtype=torch.float32, device=self.device)
                    if normuon:
                        self.neuron_state[i] = torch.zeros(rows, dtype=torch.float32, device=self.device)
                    owned.append(i)
            self._buckets.append({"W": W, "G": G, "slot": slot, "owned": owned, "plan": None})

        self._local_step = local_step
        if local_step is None:
            from . import MuonStepPlan
            beta_, nest_, lr_, wd_, steps_ = self.hyper
            opts = self._local_options
            for bk in self._buckets:
                if bk["owned"]:
                    bk["plan"] = MuonStepPlan([self.params[i] for i in bk["owned"]],
                                              [self.grads[i] for i in bk["owned"]],
                                              [self.momentum[i] for i in bk["owned"]],
                                              beta=beta_, nesterov=nest_, lr=lr_, wd=wd_, steps=steps_,
                                              **opts(bk["owned"]))

    def _local_options(self, owned):
        """Keywords of the local step for the matrices ``owned`` (none with no refinement on)."""
        if self.options is None:
            return {}
        state = None
        if self.neuron_state[owned[0]] is not None:
            state = [self.neuron_state[i] for i in owned]
        return dict(self.options, neuron_state=state)

    # ------------------------------------------------------------ collectives
    def _mine(self, flat, slot):
        return flat[self.rank * slot:(self.rank + 1) * slot]

    def _reduce_scatter_avg(self, G, slot):
        """This rank's slot of G := the group mean of every rank's slot.

        NCCL: one reduce-scatter with AVG in the gradient dtype; for bf16 each
        partial sum NCCL forms is rounded to bf16, so the mean is within about
        (world - 1) * 2^-8 of the mean of |g| of the exact mean.  Other
        backends (no reduce-scatter): an all-reduce of the gradients widened to
        fp32, the mean divided in fp32 and rounded once to the gradient dtype.
        """
        if self.dist is None:
            return
        if self._nccl:
            self.dist.reduce_scatter_tensor(self._mine(G, slot), G, op=self.dist.ReduceOp.AVG,
                                            group=self.group)
        else:
            acc = G if G.dtype == torch.float32 else G.float()
            self.dist.all_reduce(acc, op=self.dist.ReduceOp.SUM, group=self.group)
            mean = self._mine(acc, slot).div_(self.world)
            if acc is not G:
                self._mine(G, slot).copy_(mean)

    def _all_gather(self, W, slot):
        """Every rank's slot of W := its owner's; returns the pending work or None."""
        if self.dist is None:
            return None
        if self._nccl:
            return self.dist.all_gather_into_tensor(W, self._mine(W, slot), group=self.group,
                                                    async_op=True)
        chunks = list(W.split(slot))
        return self.dist.all_gather(chunks, self._mine(W, slot).clone(), group=self.group,
                                    async_op=True)

    # ------------------------------------------------------------------ step
    def step(self, lr=None, wd=None):
        """One optimizer step over the group (every rank calls it, with the same
        arguments).  ``lr`` / ``wd`` replace the constructor's values from this
        step on (a learning-rate schedule); None keeps the current one."""
        if lr is not None or wd is not None:
            b_, n_, lr_, wd_, st_ = self.hyper
            self.hyper = (b_, n_, float(lr_ if lr is None else lr), float(wd_ if wd is None else wd), st_)
            for bk in self._buckets:
                if bk["plan"] is not None:
                    bk["plan"].update(lr=self.hyper[2], wd=self.hyper[3])
        for bk in self._buckets:
            self._reduce_scatter_avg(bk["G"], bk["slot"])
        pending = []
        beta, nest, lr, wd, steps = self.hyper
        for bk in self._buckets:
            if bk["owned"]:
                if bk["plan"] is not None:
                    bk["plan"]()
                else:
                    own = bk["owned"]
                    self._local_step([self.params[i] for i in own], [self.grads[i] for i in own],
                                     [self.momentum[i] for i in own], beta, nest, lr, wd, steps,
                                     **self._local_options(own))
            work = self._all_gather(bk["W"], bk["slot"])
            if work is not None:
                pending.append(work)
        for work in pending:
            work.wait()

    # ------------------------------------------------------------ checkpoint
    def state_dict(self):
        """This rank's optimizer state: the current hyper-parameters and, for
        every matrix it owns, its momentum buffer (and NorMuon state), keyed by
        matrix index.  The weights are ``params`` (every rank holds them all)."""
        own = [i for i, m in enumerate(self.momentum) if m is not None]
        out = {"hyper": self.hyper, "shapes": list(self.shapes),
               "momentum": {i: self.momentum[i].detach().clone() for i in own}}
        if any(v is not None for v in self.neuron_state):
            out["neuron_state"] = {i: self.neuron_state[i].detach().clone() for i in own}
        return out

    def load_state_dict(self, state):
        """Restore from ``state_dict()``, or from several ranks' dicts merged
        (their ``momentum`` / ``neuron_state`` maps joined): the saving group
        may have had another size or ownership, as long as every matrix this
        rank owns is present.  Every rank calls it before its next step."""
        if [tuple(s) for s in state["shapes"]] != self.shapes:
            raise ValueError("the state is for another set of matrix shapes")
        if tuple(state["hyper"])[4] != self.hyper[4]:
            raise ValueError("the state is for another Newton-Schulz step count")
        b_, n_, lr_, wd_, st_ = (float(state["hyper"][0]), bool(state["hyper"][1]),
                                 float(state["hyper"][2]), float(state["hyper"][3]), int(state["hyper"][4]))
        has_state = any(v is not None for v in self.neuron_state)
        if has_state != ("neuron_state" in state):
            raise ValueError("NorMuon state present in one of the optimizer and the checkpoint only")
        for i, m in enumerate(self.momentum):
            if m is None:
                continue
            if i not in state["momentum"]:
                raise ValueError(f"matrix {i} is owned by this rank but missing from the state")
            m.copy_(state["momentum"][i])
            if has_state:
                self.neuron_state[i].copy_(state["neuron_state"][i])
        self.hyper = (b_, n_, lr_, wd_, st_)
        for bk in self._buckets:
            if bk["plan"] is not None:
                bk["plan"].update(beta=b_, nesterov=n_, lr=lr_, wd=wd_)
