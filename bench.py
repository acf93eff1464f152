#!/usr/bin/env python
"""Benchmark of the Muon step on B200: GPT-2-small hidden set, full muon_step.

One "step" = one full Muon update (momentum, Frobenius normalisation, five
Newton-Schulz iterations, scale and apply) of all 72 hidden matrices of GPT-2
small (12 layers x [4 x 768x768, 768x3072, 3072x768]); bf16 gradients drawn
iid N(0, 0.01^2), fp32 momentum (beta 0.95, Nesterov), lr 0.05, wd 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --ns-cases      # NS-only: batched 768x3072 and the width sweep
    python bench.py --sharded       # the data-parallel step (ShardedMuon) over the ranks

Prints one JSON line (rank 0).  `value` is matrices/s over all ranks with
inputs resident in HBM; `e2e` repeats the measurement with the gradients
copied in from pinned host memory and the updated weights copied back every
step (the copies of one step overlap the compute of its neighbours).
Per-kernel device times are taken live with CUDA events on the launching
stream (the library's timing hooks); `roofline` reports the dominant kernel
against the measured peaks in MEASURED_PEAKS.json.  After the timed region
(outside it) the same run adds: `value_sustained`, a loop of at least a
second without the timing hooks, with its own clock record; `value_graph`,
the same step recorded once in a CUDA graph and replayed (hooks off);
`step_distribution`, median / p10 / p90 of single-step times, warm and with L2
flushed before each step; `ns_768x3072`,
muon_ns_orthogonalize on 64 matrices 768x3072 (the three GEMMs and the whole
call, nominal and executed TFLOP/s); `scaled_set`, the 144-matrix 1024-wide
set's full muon_step; `refinements`, muon_step_ex with cautious weight decay
and NorMuon's per-neuron rescale on the GPT-2-small set; `square_sweep`, the
square width sweep m = 256 .. 4096 (batch 64 (768/m)^2).
`--impl reference` times the fp64 CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Muon NS-5 matrices/s and TFLOP/s (% of B200 BF16 peak), GPT-2-small set"
UNIT = "matrices/s"
WORKLOAD = ("GPT-2-small hidden set: 12 layers x (4x 768x768, 768x3072, 3072x768) = 72 matrices; "
            "bf16 grads iid N(0,1e-2^2), fp32 momentum beta=0.95 Nesterov, T=5, lr 0.05, wd 0")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
BAD_REASONS = {"hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"}
REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sharded", action="store_true",
                    help="time ShardedMuon (reduce-scatter, local step, all-gather) over the ranks "
                         "instead of independent replicas")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the sustained loop and the NS-only / scaled-set measurements")
    ap.add_argument("--ns-cases", action="store_true",
                    help="instead of the step benchmark: muon_ns_orthogonalize (bf16) on the "
                         "batched 768x3072 case and the square width sweep, one JSON line each")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- workload
def gpt2_shapes():
    from newton_schulz_12_b200 import workloads
    return workloads.gpt2_small_shapes()


def nominal_flops(shapes, steps=5):
    """steps * (4 m^2 n + 2 m^3) per matrix, m = min, n = max."""
    tot = 0
    for r, c in shapes:
        m, n = min(r, c), max(r, c)
        tot += steps * (4 * m * m * n + 2 * m ** 3)
    return tot


PAIR_TILE = 256  # rows x columns of one tensor-core pair tile
K_STAGE = 64     # K of one operand stage


def executed_flops(shapes, steps=5):
    """FLOPs the tensor cores execute per call: whole 256 x 256 pair tiles
    (padding included), X X^T and A A only on the tiles on or above the
    diagonal, B X on every tile; K rounded up to the 64-deep stage."""
    tot = 0
    for r, c in shapes:
        m, n = min(r, c), max(r, c)
        tm = -(-m // PAIR_TILE)
        tn = -(-n // PAIR_TILE)
        sym = tm * (tm + 1) // 2
        kn = -(-n // K_STAGE) * K_STAGE
        km = -(-m // K_STAGE) * K_STAGE
        tile = 2 * PAIR_TILE * PAIR_TILE
        tot += steps * tile * (sym * kn + sym * km + tm * tn * km)
    return tot


def stage_work(shapes):
    """Algorithmic work of one launch of each kernel kind over the whole set.

    GEMMs: nominal FLOPs (X X^T: 2 m^2 n, A A: 2 m^3, B X: 2 m^2 n).
    Memory-bound kernels: bytes that must cross HBM per element -- prep
    g(2)+buf(4) read, buf(4) and the pair bf16 hi(2) + int8 lo(1) of u
    written = 13 B; apply W(4) + O as hi(2)+lo(1) read, W(4) written = 11 B;
    (fp32 and stand-alone paths) momentum 10 B, cast 10 B.  The per-matrix
    scale reads one fp64 partial per prep block.  The last step's fused
    BX + apply reads X's pair (3 B) and W (4 B), writes W (4 B) per element
    and reads B (2 B per element of the m x m matrix): HBM-bound.
    """
    elems = sum(r * c for r, c in shapes)
    g = sum(2 * min(r, c) ** 2 * max(r, c) for r, c in shapes)
    p = sum(2 * min(r, c) ** 3 for r, c in shapes)
    prep_blocks = sum(-(-r // 64) * -(-c // 128) for r, c in shapes)
    return {
        "gram": ("tensor", g), "poly": ("tensor", p), "bx": ("tensor", g),
        "bx_apply": ("hbm", 11 * elems + sum(2 * min(r, c) ** 2 for r, c in shapes)),
        "prep": ("hbm", 13 * elems), "scale": ("hbm", 8 * prep_blocks + 4 * len(shapes)),
        "flat": ("hbm", 10 * elems), "cast": ("hbm", 10 * elems), "out": ("hbm", 11 * elems),
    }


# ------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    def __init__(self, torch_device):
        self.samples, self.reasons, self.max_mhz, self.err = [], set(), None, None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(torch_device)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = f"nvml unavailable: {e}"
            self.h = None

    def _run(self):
        nv = self.nvml
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = get_reasons(self.h)
                for b, name in REASON_BITS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception as e:  # pragma: no cover
                self.err = str(e)
                break
            time.sleep(0.005)

    def __enter__(self):
        if self.h is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self):
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None,
               "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
               "samples": len(self.samples)}
        if self.err:
            out["note"] = self.err
        return out


# ---------------------------------------------------------------- oracle legs
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_matrix_step(shape, idx):
    """One fp64 oracle Muon step of one GPT-2 hidden matrix (seeded as in the GPU run)."""
    import numpy as np
    from newton_schulz_12_b200 import workloads
    from oracle import muon as oracle
    Ws, Gs = workloads.muon_set([shape], step=0, grad_seed=1000 + idx, w_seed=2000 + idx)
    W = Ws[0].double().numpy()
    g = Gs[0].float().numpy()
    return oracle.muon_step(W, g, np.zeros(shape), beta=0.95, nesterov=True, lr=0.05, wd=0.0)


def cpu_baseline(shapes, budget_s=12.0):
    """The oracle on whole layers (4 square + wide + tall) until ~budget_s of CPU time."""
    layer = shapes[:6]
    done, t0 = 0, time.perf_counter()
    while True:
        for i, s in enumerate(layer):
            oracle_matrix_step(s, i)
        done += len(layer)
        if time.perf_counter() - t0 >= budget_s or done >= len(shapes):
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{done // 6} of 12 GPT-2-small layers ({done} of 72 matrices), full Muon "
                      f"step in fp64 (numpy, BLAS matmul), {dt:.1f} s"}


def run_reference(args):
    """`--impl reference`: the fp64 oracle as it stands, on host cores, rank 0 only.

    A step is one whole GPT-2-small layer (its 6 hidden matrices: 4x 768x768,
    768x3072, 3072x768), the same mix and unit as the GPU arm's 72-matrix set."""
    rank = rank_env()[1]
    if rank != 0:
        return
    shapes = gpt2_shapes()
    layer = shapes[:6]

    def one_layer():
        for i, s in enumerate(layer):
            oracle_matrix_step(s, i)

    for _ in range(args.warmup):
        one_layer()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one_layer()
    dt = time.perf_counter() - t0
    value = len(layer) * args.steps / dt
    cores = _blas_threads()
    sample = (f"each step = one whole GPT-2-small layer (4x 768x768, 768x3072, 3072x768), "
              f"full Muon step in fp64 numpy; {args.steps} layers timed")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * dt / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "matrices_per_step": len(layer),
                   "parallelism": "none (host cores)"},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ranks
def rank_env():
    """(world, rank, local_rank) from the torch.distributed launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value, device):
    """Maximum of a per-rank float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank, world, steps, ms):
    """Whole-job throughput: units processed by all ranks over the slowest rank's time."""
    return units_per_rank * world * steps / (ms / 1000.0)


# ------------------------------------------------------------------ our arm
def traffic_record():
    """Per-launch DRAM bytes of the dominant kernel from a committed ncu summary, if current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except Exception:
        return None
    h = hashlib.sha256()
    for name in rec.get("sources", []):
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    if h.hexdigest() != rec.get("sources_sha256"):
        return None
    return rec


# ------------------------------------------------ measurements after the timed region
def time_steps(fn, n, stream):
    """Device time (ms) of n calls of fn on `stream`, CUDA events, synchronised on both sides."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(n):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def measure_sustained(step, stream, dev, ms_hint, units, min_s=1.5):
    """The same step in a loop of at least `min_s` seconds, timing hooks off:
    the steady-state rate under the power cap, with its clock record."""
    n = max(50, int(min_s * 1000.0 / max(ms_hint, 1e-3)) + 1)
    for _ in range(3):
        step()
    with ClockSampler(dev) as clocks:
        ms = time_steps(step, n, stream)
    c = clocks.summary()
    out = {"value": units * n / (ms / 1000.0), "unit": UNIT, "steps": n, "ms_per_step": ms / n,
           "seconds": ms / 1000.0, "clocks": c}
    if c.get("sm_mhz"):
        out["ms_x_sm_ghz"] = ms / n * c["sm_mhz"] / 1000.0
    return out


def measure_step_distribution(step, stream, dev, reps=50):
    """Per-step device times (timing hooks off), each step between its own
    pair of events: median, p10 and p90 over `reps` steps, once warm (inputs
    already larger than L2) and once with L2 flushed before every step (a
    256 MB buffer, twice L2, written between the steps, outside their events)."""
    import torch
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)
    out = {}
    for kind in ("warm", "l2_flushed"):
        for _ in range(3):
            step()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(reps)]
        torch.cuda.synchronize(dev)
        for a, b in evs:
            if kind == "l2_flushed":
                flush.fill_(1.0)
            a.record(stream)
            step()
            b.record(stream)
        torch.cuda.synchronize(dev)
        t = sorted(a.elapsed_time(b) for a, b in evs)
        q = lambda f: t[min(len(t) - 1, int(round(f * (len(t) - 1))))]  # noqa: E731
        out[kind] = {"median_ms": q(0.5), "p10_ms": q(0.1), "p90_ms": q(0.9), "steps": reps}
    del flush
    return out


def measure_ns_768x3072(dev, peaks, reps=20):
    """muon_ns_orthogonalize (bf16) on 64 matrices 768 x 3072: the three GEMMs
    (from the timing hooks) and the whole call, nominal and executed TFLOP/s."""
    import torch
    import newton_schulz_12_b200 as nsb
    m, n, batch = 768, 3072, 64
    g = torch.Generator(device="cpu").manual_seed(3000 + m)
    xs = [torch.randn(m, n, generator=g).to(torch.bfloat16).to(dev) for _ in range(batch)]
    stream = torch.cuda.current_stream(dev)
    plan = nsb.MuonNsPlan(xs)
    for _ in range(3):
        plan(stream)
    with ClockSampler(dev) as clocks:
        nsb.muon_profile_begin()
        ms = time_steps(lambda: plan(stream), reps, stream)
        prof = nsb.muon_profile_end()
    if nsb.muon_get_status() != 0:
        raise RuntimeError("device status in the 768x3072 case: " + nsb.muon_last_error())
    nominal = nominal_flops([(m, n)] * batch)
    executed = executed_flops([(m, n)] * batch)
    gemm_ms = sum(prof[k][0] for k in ("gram", "poly", "bx")) / reps
    call_ms = ms / reps
    out = {"batch": batch, "m": m, "n": n, "reps": reps, "call_ms": call_ms, "gemm_ms": gemm_ms,
           "nominal_gflop": nominal / 1e9, "executed_gflop": executed / 1e9,
           "gemm_tflops_nominal": nominal / gemm_ms / 1e9, "gemm_tflops_executed": executed / gemm_ms / 1e9,
           "call_tflops_nominal": nominal / call_ms / 1e9, "call_tflops_executed": executed / call_ms / 1e9,
           "peak": peaks["bf16_tflops"],
           "per_kernel_us": {k: v[0] / v[1] * 1e3 for k, v in prof.items() if v[1]},
           "clocks": clocks.summary()}
    out["gemm_frac_nominal"] = out["gemm_tflops_nominal"] / peaks["bf16_tflops"]
    out["gemm_frac_executed"] = out["gemm_tflops_executed"] / peaks["bf16_tflops"]
    del xs
    return out


def measure_graph(plan, dev, ms_hint, units, min_s=1.0):
    """The same step recorded once in a CUDA graph (MuonStepPlan.capture) and
    replayed for at least `min_s` seconds, timing hooks off: the launch gaps
    of 17 stream launches per step mostly disappear.  capture() itself runs
    one step (outside the timing)."""
    import torch
    import newton_schulz_12_b200 as nsb
    plan.capture()
    stream = torch.cuda.current_stream(dev)
    n = max(50, int(min_s * 1000.0 / max(ms_hint, 1e-3)) + 1)
    for _ in range(3):
        plan.replay()
    with ClockSampler(dev) as clocks:
        ms = time_steps(plan.replay, n, stream)
    if nsb.muon_get_status(stream) != 0:
        raise RuntimeError("device status in the graph replay: " + nsb.muon_last_error())
    return {"value": units * n / (ms / 1000.0), "unit": UNIT, "steps": n, "ms_per_step": ms / n,
            "clocks": clocks.summary()}


def measure_refinements(W, G, M, shapes, stream, dev, steps=20):
    """muon_step_ex on the GPT-2 set with both refinements on: cautious weight
    decay (wd 0.01) and NorMuon's per-neuron rescale (beta2 0.95); the
    rescale needs every row's norm first, so every update takes the apply
    pass (no fused apply).  Same tensors as the main run (W and momentum keep
    evolving)."""
    import torch
    import newton_schulz_12_b200 as nsb
    V = [torch.zeros(r, device=dev) for r, _ in shapes]

    def step():
        nsb.muon_step_ex(W, G, M, wd=0.01, cautious_wd=True, neuron_state=V, beta2=0.95, stream=stream)

    for _ in range(3):
        step()
    with ClockSampler(dev) as clocks:
        nsb.muon_profile_begin()
        ms = time_steps(step, steps, stream)
        prof = nsb.muon_profile_end()
    if nsb.muon_get_status(stream) != 0:
        raise RuntimeError("device status in the refinements run: " + nsb.muon_last_error())
    per = ms / steps
    return {"options": "cautious_wd + NorMuon (beta2 0.95), wd 0.01", "steps": steps,
            "ms_per_step": per, "value": len(shapes) / (per / 1000.0), "unit": UNIT,
            "per_kernel_us": {k: v[0] / v[1] * 1e3 for k, v in prof.items() if v[1]},
            "launches_per_step": sum(v[1] for v in prof.values()) / steps,
            "clocks": clocks.summary()}


def measure_square_sweep(dev, peaks, reps=10):
    """muon_ns_orthogonalize (bf16) on the square width sweep: m in {256 .. 4096}
    with batch 64 (768/m)^2 (>= 1), bf16 N(0, 1) drawn on the device; GEMM
    and whole-call TFLOP/s, nominal and executed, per width.  The call goes
    through MuonNsPlan (arguments marshalled once); `call_ms_graph` is the same
    call replayed from a CUDA graph."""
    import torch
    import newton_schulz_12_b200 as nsb
    from newton_schulz_12_b200 import workloads
    stream = torch.cuda.current_stream(dev)
    out = []
    for m, batch in workloads.sweep_cases():
        g = torch.Generator(device=dev).manual_seed(3000 + m)
        xs = [torch.randn(m, m, generator=g, device=dev).to(torch.bfloat16) for _ in range(batch)]
        plan = nsb.MuonNsPlan(xs)
        for _ in range(2):
            plan(stream)
        nsb.muon_profile_begin()
        ms = time_steps(lambda: plan(stream), reps, stream)
        prof = nsb.muon_profile_end()
        if nsb.muon_get_status() != 0:
            raise RuntimeError(f"device status in the sweep at m={m}: " + nsb.muon_last_error())
        gs = torch.cuda.Stream(dev)
        plan.capture(gs)
        with torch.cuda.stream(gs):
            ms_graph = time_steps(plan.replay, reps, gs)
        del plan
        nominal = nominal_flops([(m, m)] * batch)
        executed = executed_flops([(m, m)] * batch)
        gemm_ms = sum(prof[k][0] for k in ("gram", "poly", "bx")) / reps
        out.append({"m": m, "batch": batch, "call_ms": ms / reps, "call_ms_graph": ms_graph / reps,
                    "gemm_ms": gemm_ms,
                    "gemm_tflops_nominal": nominal / gemm_ms / 1e9,
                    "gemm_tflops_executed": executed / gemm_ms / 1e9,
                    "call_tflops_nominal": nominal / (ms / reps) / 1e9,
                    "gemm_frac_executed": executed / gemm_ms / 1e9 / peaks["bf16_tflops"]})
        del xs
    return out


def measure_scaled_set(dev, peaks, steps=10):
    """Full muon_step over the 144-matrix 1024-wide set (24 layers x [4x 1024^2,
    1024x4096, 4096x1024]), bf16 grads N(0, 0.01^2), fp32 W N(0, 0.02^2),
    momentum zeros, wd 0.01.  Inputs drawn on the device (seeded)."""
    import torch
    import newton_schulz_12_b200 as nsb
    from newton_schulz_12_b200 import workloads
    shapes = workloads.scaled_shapes()
    counts = [r * c for r, c in shapes]
    total = sum(counts)
    offs = [0]
    for k in counts:
        offs.append(offs[-1] + k)
    g = torch.Generator(device=dev).manual_seed(5)
    W_flat = torch.randn(total, generator=g, device=dev) * 0.02
    G_flat = (torch.randn(total, generator=g, device=dev) * 0.01).to(torch.bfloat16)
    M_flat = torch.zeros(total, device=dev)
    view = lambda flat, i: flat[offs[i]:offs[i + 1]].view(shapes[i])  # noqa: E731
    plan = nsb.MuonStepPlan([view(W_flat, i) for i in range(len(shapes))],
                            [view(G_flat, i) for i in range(len(shapes))],
                            [view(M_flat, i) for i in range(len(shapes))], wd=0.01)
    stream = torch.cuda.current_stream(dev)
    for _ in range(3):
        plan(stream)
    with ClockSampler(dev) as clocks:
        ms = time_steps(lambda: plan(stream), steps, stream)
    if nsb.muon_get_status(stream) != 0:
        raise RuntimeError("device status in the scaled set: " + nsb.muon_last_error())
    per = ms / steps
    flops = nominal_flops(shapes)
    out = {"matrices": len(shapes), "steps": steps, "ms_per_step": per,
           "value": len(shapes) / (per / 1000.0), "unit": UNIT,
           "tflops_nominal": flops / per / 1e9, "pct_of_bf16_peak": 100.0 * flops / per / 1e9 / peaks["bf16_tflops"],
           "l2": "inputs far larger than L2 (W 1.2 GB, momentum 1.2 GB, grads 0.6 GB); no flush",
           "clocks": clocks.summary()}
    del plan, W_flat, G_flat, M_flat
    return out


def run_ours(args):
    import torch
    import torch.distributed as dist

    import newton_schulz_12_b200 as nsb
    from newton_schulz_12_b200 import workloads

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    peaks, peak_src = load_peaks()
    shapes = gpt2_shapes()
    counts = [r * c for r, c in shapes]
    total = sum(counts)
    offs = [0]
    for n in counts:
        offs.append(offs[-1] + n)
    # one flat allocation per tensor kind; every matrix a view (all 16-byte aligned)
    Ws, Gs = workloads.muon_set(shapes, step=0)
    W_flat = torch.empty(total, dtype=torch.float32, device=dev)
    G_flat = torch.empty(total, dtype=torch.bfloat16, device=dev)
    M_flat = torch.zeros(total, dtype=torch.float32, device=dev)
    for i in range(len(shapes)):
        W_flat[offs[i]:offs[i + 1]].copy_(Ws[i].reshape(-1))
        G_flat[offs[i]:offs[i + 1]].copy_(Gs[i].reshape(-1))
    W = [W_flat[offs[i]:offs[i + 1]].view(shapes[i]) for i in range(len(shapes))]
    G = [G_flat[offs[i]:offs[i + 1]].view(shapes[i]) for i in range(len(shapes))]
    M = [M_flat[offs[i]:offs[i + 1]].view(shapes[i]) for i in range(len(shapes))]
    stream = torch.cuda.current_stream(dev)

    plan = nsb.MuonStepPlan(W, G, M, beta=0.95, nesterov=True, lr=0.05, wd=0.0, steps=5)

    def step():
        plan(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if nsb.muon_get_status(stream) != 0:
        raise RuntimeError("device status after warm-up: " + nsb.muon_last_error())

    # ---- timed region: inputs resident in HBM
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        nsb.muon_profile_begin()
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize(dev)
    prof = nsb.muon_profile_end()
    barrier()
    ms = max_over_ranks(start.elapsed_time(end), dev)
    if nsb.muon_get_status(stream) != 0:
        raise RuntimeError("device status after timed region: " + nsb.muon_last_error())
    launches = sum(n for _, n in prof.values())

    # ---- end to end: pinned host grads in, updated weights out, every step.
    # The copies overlap the neighbouring steps' compute, as a training loop
    # would: step k's grads go into one of two device buffers on a copy-in
    # stream while step k-1 runs; after step k the weights are copied to a
    # device staging buffer (step k+1 then updates W in place) and read back
    # to the host on a copy-out stream while step k+1 runs.
    G_host = G_flat.cpu().pin_memory()
    W_host = torch.empty(total, dtype=torch.float32).pin_memory()
    G_dev = [G_flat, torch.empty_like(G_flat)]
    plans = []
    for g in G_dev:
        views = [g[offs[i]:offs[i + 1]].view(shapes[i]) for i in range(len(shapes))]
        plans.append(nsb.MuonStepPlan(W, views, M, beta=0.95, nesterov=True, lr=0.05, wd=0.0, steps=5))
    W_stage = torch.empty_like(W_flat)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    g_ready = [torch.cuda.Event(), torch.cuda.Event()]
    g_free = [torch.cuda.Event(), torch.cuda.Event()]
    staged, out_done = torch.cuda.Event(), torch.cuda.Event()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = args.steps
    barrier()
    torch.cuda.synchronize(dev)
    e_start.record(stream)
    s_in.wait_event(e_start)
    s_out.wait_event(e_start)
    for k in range(e2e_steps):
        j = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(g_free[j])  # step k-2 is done with this buffer
            G_dev[j].copy_(G_host, non_blocking=True)
            g_ready[j].record(s_in)
        stream.wait_event(g_ready[j])
        plans[j](stream)
        g_free[j].record(stream)
        if k >= 1:
            stream.wait_event(out_done)  # step k-1's read-back is done with the staging buffer
        W_stage.copy_(W_flat, non_blocking=True)
        staged.record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(staged)
            W_host.copy_(W_stage, non_blocking=True)
            out_done.record(s_out)
    stream.wait_event(out_done)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e_ms = max_over_ranks(e_start.elapsed_time(e_end), dev)
    if nsb.muon_get_status(stream) != 0:
        raise RuntimeError("device status after the end-to-end run: " + nsb.muon_last_error())

    nmat = len(shapes) * world
    value = job_throughput(len(shapes), world, args.steps, ms)
    flops_step = nominal_flops(shapes)
    tflops = flops_step * world * args.steps / (ms / 1000.0) / 1e12

    # ---- per-kernel roofline from the live event timings (rank 0's)
    work = stage_work(shapes)
    kernels = {}
    for kind, (tot_ms, n) in prof.items():
        if n == 0:
            continue
        per = tot_ms / n
        entry = {"launches": n, "ms_per_launch": per, "ms_per_step": tot_ms / args.steps}
        if kind in work:
            bound, amount = work[kind]
            if bound == "tensor":
                ach = amount / (per / 1000.0) / 1e12
                entry.update(bound="tensor", achieved=ach, unit="TFLOP/s",
                             frac=ach / peaks["bf16_tflops"])
            else:
                ach = amount / (per / 1000.0) / 1e9
                entry.update(bound="hbm", achieved=ach, unit="GB/s", frac=ach / peaks["hbm_gbs"])
        kernels[kind] = entry
    dom = max((k for k in kernels if k in work), key=lambda k: kernels[k]["ms_per_step"])
    d = kernels[dom]
    trec = traffic_record()
    traffic = None
    if trec and trec.get("kernel_kind") == dom:
        traffic = trec.get("bytes_per_launch")
    roofline = {"bound": d["bound"], "achieved": d["achieved"],
                "peak": peaks["bf16_tflops"] if d["bound"] == "tensor" else peaks["hbm_gbs"],
                "unit": d["unit"], "frac": d["frac"], "traffic": traffic, "kernel": dom,
                "peak_source": f"{peak_src} ({'bf16 burst' if d['bound'] == 'tensor' else 'copy'})"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "matrices_per_step": len(shapes) * world,
                       "parallelism": f"replicas x{world} (one independent 72-matrix set per GPU)",
                       "l2": "inputs larger than L2 (W 340 MB + momentum 340 MB + grads 170 MB "
                             "per GPU, plus a 600 MB workspace); no flush"},
            "tflops": tflops,
            "pct_of_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
            "pct_of_bf16_peak_sustained": 100.0 * tflops / peaks["bf16_tflops_sustained"],
            "roofline": roofline,
            "kernels": kernels,
            "gpu_launches": launches,
            "e2e": {"value": job_throughput(len(shapes), world, e2e_steps, e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": G_host.numel() * G_host.element_size(),
                    "d2h_bytes_per_step": W_host.numel() * W_host.element_size()},
            "clocks": clocks.summary(),
        }
        if world == 1 and not args.no_extras:
            line["value_sustained"] = measure_sustained(step, stream, dev, ms / args.steps, len(shapes))
            line["value_graph"] = measure_graph(plan, dev, ms / args.steps, len(shapes))
            line["step_distribution"] = measure_step_distribution(step, stream, dev)
            line["refinements"] = measure_refinements(W, G, M, shapes, stream, dev)
            line["ns_768x3072"] = measure_ns_768x3072(dev, peaks)
            line["square_sweep"] = measure_square_sweep(dev, peaks)
            del W_flat, G_flat, M_flat, W, G, M, plan, plans, G_dev, W_stage
            torch.cuda.empty_cache()
            line["scaled_set"] = measure_scaled_set(dev, peaks)
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(shapes)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ------------------------------------------------------- data-parallel step
def run_sharded(args):
    """`--sharded`: ShardedMuon over the ranks -- reduce-scatter of the bf16
    gradients by owner (NCCL), the local muon_step on the owned matrices, and
    an asynchronous all-gather of the updated fp32 weights per bucket -- on the
    72-matrix GPT-2-small set.  A step updates the whole set once, so the work
    per step is fixed as ranks are added (strong scaling)."""
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import newton_schulz_12_b200 as nsb
    from newton_schulz_12_b200 import workloads
    from newton_schulz_12_b200.sharded import ShardedMuon

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    if "MASTER_PORT" not in os.environ:
        import socket
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            os.environ["MASTER_PORT"] = str(sk.getsockname()[1])
    dist.init_process_group("nccl", rank=rank, world_size=world, timeout=timedelta(seconds=120),
                            device_id=dev)
    peaks, _ = load_peaks()
    shapes = gpt2_shapes()
    sm = ShardedMuon(shapes, device=dev, buckets=2, beta=0.95, nesterov=True, lr=0.05, wd=0.0, steps=5)
    Ws, Gs = workloads.muon_set(shapes, step=0)
    for i in range(len(shapes)):
        sm.params[i].copy_(Ws[i])
        sm.grads[i].copy_(Gs[i])
    stream = torch.cuda.current_stream(dev)
    for _ in range(max(3, args.warmup)):
        sm.step()
    torch.cuda.synchronize(dev)
    dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clocks:
        nsb.muon_profile_begin()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            sm.step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        prof = nsb.muon_profile_end()
    dist.barrier()
    ms = max_over_ranks(a.elapsed_time(b), dev)
    kern_ms = sum(t for t, _ in prof.values()) / args.steps
    kern_max = max_over_ranks(kern_ms, dev)
    if nsb.muon_get_status(stream) != 0:
        raise RuntimeError("device status in the sharded run: " + nsb.muon_last_error())
    owned = sum(1 for o in sm.owner if o == rank)
    if rank == 0:
        per = ms / args.steps
        line = {
            "metric": METRIC, "value": len(shapes) / (per / 1000.0), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": per,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "matrices_per_step": len(shapes),
                       "parallelism": f"sharded dp{world}: reduce-scatter of bf16 grads by owner "
                                      "(NCCL AVG), local muon_step, async all-gather of fp32 W per "
                                      "bucket (2 buckets)",
                       "matrices_owned_rank0": owned},
            "kernel_ms_per_step_max_rank": kern_max,
            "comm_and_host_ms_per_step": per - kern_max,
            "tflops": nominal_flops(shapes) / per / 1e9,
            "gpu_launches": sum(n for _, n in prof.values()),
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    dist.barrier()
    dist.destroy_process_group()


# ------------------------------------------------------- NS-only case sweep
NS_CASES = [  # (label, m, n, batch): the batched 768x3072 case, then m in {256..4096} with
              # batch 64 (768/m)^2 rounded, at least 1
    ("768x3072 x64", 768, 3072, 64),
    ("256^2 x576", 256, 256, 576), ("512^2 x144", 512, 512, 144), ("768^2 x64", 768, 768, 64),
    ("1024^2 x36", 1024, 1024, 36), ("2048^2 x9", 2048, 2048, 9), ("4096^2 x2", 4096, 4096, 2),
]


def run_ns_cases(args):
    """Per case: the whole muon_ns_orthogonalize call and its three GEMM kernels
    (device time from the library's timing hooks) against the bf16 peak."""
    import torch
    import newton_schulz_12_b200 as nsb
    peaks, peak_src = load_peaks()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    for label, m, n, batch in NS_CASES:
        g = torch.Generator(device="cpu").manual_seed(3000 + m)
        xs = [torch.randn(m, n, generator=g).to(torch.bfloat16).to(dev) for _ in range(batch)]
        flops = nominal_flops([(m, n)] * batch)
        plan = nsb.MuonNsPlan(xs)
        for _ in range(args.warmup):
            plan()
        torch.cuda.synchronize()
        reps = max(3, min(args.steps, 50))
        nsb.muon_profile_begin()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(reps):
            plan()
        t1.record()
        torch.cuda.synchronize()
        prof = nsb.muon_profile_end()
        if nsb.muon_get_status() != 0:
            raise SystemExit(f"device status error in case {label}")
        call_ms = t0.elapsed_time(t1) / reps
        gemm_ms = sum(prof[k][0] for k in ("gram", "poly", "bx")) / reps
        x_bytes = batch * m * n * 2
        print(json.dumps({
            "case": label, "m": m, "n": n, "batch": batch, "reps": reps,
            "nominal_gflop": flops / 1e9,
            "call_ms": call_ms, "tflops_call": flops / call_ms / 1e9,
            "gemm_ms": gemm_ms, "tflops_gemm": flops / gemm_ms / 1e9,
            "gemm_frac_of_peak": flops / gemm_ms / 1e9 / peaks["bf16_tflops"],
            "peak": peaks["bf16_tflops"], "peak_source": f"{peak_src} (bf16 burst)",
            "per_kernel_us": {k: v[0] / v[1] * 1e3 for k, v in prof.items() if v[1]},
            "l2": "X %.0f MB (%s the 126 MB L2), workspace larger; no flush" % (
                x_bytes / 1e6, "above" if x_bytes > 126e6 else "below"),
        }), flush=True)
        del xs
        torch.cuda.empty_cache()


def main():
    args = parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.ns_cases:
        run_ns_cases(args)
    elif args.sharded and args.impl == "ours":
        run_sharded(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
