"""Single-kernel workloads for profiler captures (ncu) of the library's kernels.

    python -m newton_schulz_12_b200.profile_case {bx,gram,poly,step,bxapply,stepex} [--reps N]

Each case allocates its operands once (seeded, synthetic), then calls one C-ABI
entry point `reps` times and synchronises, so a profiler can skip the first
(warm-up) launch and capture the next.  Sizes are the GPT-2-small ones and
exceed the 126 MB L2, so DRAM counters are meaningful, while staying far
below the device's memory:

  bx    X' = aX + BX over 24 matrices 768x3072 (B 768x768)      ~310 MB
  gram  A = X X^T over 24 matrices 768x3072                      ~140 MB
  poly  B = bA + cA^2 over 72 matrices 768x768                   ~170 MB
  step  one full muon_step over the 72-matrix GPT-2-small set    ~1.7 GB
  bxapply  the last step's BX with the apply fused (muon_bx_apply_bf16)
        over 12 matrices 768x3072 with tall fp32 W (3072x768)     ~400 MB
  stepex   muon_step_ex (cautious decay + NorMuon) over the GPT-2 set ~1.7 GB
"""
from __future__ import annotations

import argparse

import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import workloads


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("case", choices=["bx", "gram", "poly", "step", "bxapply", "stepex"])
    ap.add_argument("--reps", type=int, default=2)
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    g = torch.Generator(device="cpu").manual_seed(1)
    if args.case == "bx":
        B = (torch.randn(24, 768, 768, generator=g) / 768 ** 0.5).to(torch.bfloat16).to(dev)
        X = (torch.randn(24, 768, 3072, generator=g) / 3072 ** 0.5).to(dev)
        hi = X.to(torch.bfloat16)
        lo = torch.zeros(X.shape, dtype=torch.int8, device=dev)  # the int8 part of the pair
        out = torch.empty_like(hi)
        for _ in range(args.reps):
            nsb.muon_bx_bf16(B, hi, lo, Xhi_out=out)
    elif args.case == "gram":
        X = torch.randn(24, 768, 3072, generator=g).to(torch.bfloat16).to(dev)
        A = torch.empty(24, 768, 768, dtype=torch.bfloat16, device=dev)
        for _ in range(args.reps):
            nsb.muon_gram_bf16(X, A)
    elif args.case == "poly":
        G = torch.randn(72, 768, 768, generator=g) / 768 ** 0.5
        A = ((G + G.transpose(1, 2)) / 2).to(torch.bfloat16).to(dev)
        B = torch.empty_like(A)
        for _ in range(args.reps):
            nsb.muon_poly_bf16(A, B=B)
    elif args.case == "bxapply":
        B = (torch.randn(12, 768, 768, generator=g) / 768 ** 0.5).to(torch.bfloat16).to(dev)
        X = (torch.randn(12, 768, 3072, generator=g) / 3072 ** 0.5).to(dev)
        hi = X.to(torch.bfloat16)
        lo = torch.zeros(X.shape, dtype=torch.int8, device=dev)
        W = [(torch.randn(3072, 768, generator=g) * 0.02).to(dev) for _ in range(12)]
        for _ in range(args.reps):
            nsb.muon_bx_apply_bf16(B, hi, lo, W, tall=True, wd=0.01)
    else:
        shapes = workloads.gpt2_small_shapes()
        Ws, Gs = workloads.muon_set(shapes)
        W = [w.to(dev) for w in Ws]
        G2 = [x.to(dev) for x in Gs]
        M = [torch.zeros_like(w) for w in W]
        V = [torch.zeros(r, device=dev) for r, _ in shapes]
        for _ in range(args.reps):
            if args.case == "stepex":
                nsb.muon_step_ex(W, G2, M, wd=0.01, cautious_wd=True, neuron_state=V)
            else:
                nsb.muon_step(W, G2, M)
    torch.cuda.synchronize()
    rc = nsb.muon_get_status()
    if rc != 0:
        raise SystemExit(f"device status {rc}: {nsb.muon_last_error()}")
    print(f"{args.case}: ok")


if __name__ == "__main__":
    main()
