"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle legs.

This module holds no arithmetic of the Muon method: only shapes and random
numbers.  Everything is drawn on the CPU with ``torch.Generator`` in fp32 and
cast afterwards, so the GPU path and the fp64 oracle receive identical bits.

Workloads (shapes of the NanoGPT speedrun's GPT-2 small, 124M parameters,
width m = 768 -- "The NanoGPT speedrun", paragraph "Six records account for
most of the speedup", record #3):

* ``gpt2_small_shapes``: 12 layers x (4 attention 768x768, 768x3072 MLP-in,
  3072x768 MLP-out) = 72 hidden matrices, in layer order.
* ``scaled_shapes``: 24 layers x (4 1024x1024, 1024x4096, 4096x1024) = 144.
* ``sweep_cases``: square widths {256..4096} with batch 64*(768/m)^2 (>= 1).
"""
from __future__ import annotations

import torch


def gpt2_small_shapes(layers=12, width=768):
    shapes = []
    for _ in range(layers):
        shapes += [(width, width)] * 4
        shapes += [(width, 4 * width), (4 * width, width)]
    return shapes


def scaled_shapes(layers=24, width=1024):
    return gpt2_small_shapes(layers, width)


def sweep_cases():
    """(m, batch) pairs of the square width sweep, batch = round(64*(768/m)^2) >= 1."""
    out = []
    for m in (256, 512, 768, 1024, 2048, 4096):
        out.append((m, max(1, int(round(64 * (768 / m) ** 2)))))
    return out


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def gaussian(shape, std=1.0, seed=0, dtype=torch.float32):
    """iid N(0, std^2) drawn in fp32 on the CPU, then cast to ``dtype``."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(dtype)


def _orthonormal_columns(rows, k, gen):
    """Q factor (rows x k) of a seeded Gaussian, sign-fixed by diag(R)."""
    q, r = torch.linalg.qr(torch.randn(rows, k, generator=gen, dtype=torch.float64))
    d = torch.sign(torch.diagonal(r))
    d[d == 0] = 1.0
    return q * d


def hard_spectrum(rows, cols, seed, spike=False, spike_rank=4, spike_factor=100.0,
                  scale=1e-2, dtype=torch.bfloat16):
    """U diag(s) V^T with s = 10^(-4u), u ~ U(0,1) (log-uniform in [1e-4, 1]).

    With ``spike``, the ``spike_rank`` largest singular values are multiplied by
    ``spike_factor``.  The result is scaled by ``scale`` and cast to ``dtype``.
    """
    gen = _gen(seed)
    k = min(rows, cols)
    U = _orthonormal_columns(rows, k, gen)
    V = _orthonormal_columns(cols, k, gen)
    u = torch.rand(k, generator=gen, dtype=torch.float64)
    s, _ = torch.sort(10.0 ** (-4.0 * u), descending=True)
    if spike:
        s[:spike_rank] *= spike_factor
    G = (U * s) @ V.T
    return (G * scale).to(torch.float32).to(dtype)


def spiked_indices(count, fraction=0.05, seed=77):
    """round(fraction*count) distinct matrix indices, seeded."""
    n = int(round(fraction * count))
    perm = torch.randperm(count, generator=_gen(seed))
    return sorted(int(i) for i in perm[:n])


def muon_set(shapes, step=0, grad_std=1e-2, w_std=2e-2, hard=False,
             grad_seed=1000, w_seed=2000):
    """Per-matrix (W fp32, grad bf16) for the Muon-step workloads.

    grad_i is seeded ``grad_seed + i + 100*step``; W_i is seeded
    ``w_seed + i``.  With ``hard`` the gradients have log-uniform spectra and
    5 % of the matrices carry a x100 rank-4 spike.
    """
    spikes = set(spiked_indices(len(shapes))) if hard else set()
    Ws, Gs = [], []
    for i, (r, c) in enumerate(shapes):
        Ws.append(gaussian((r, c), w_std, w_seed + i))
        seed = grad_seed + i + 100 * step
        if hard:
            Gs.append(hard_spectrum(r, c, seed, spike=(i in spikes), scale=grad_std))
        else:
            Gs.append(gaussian((r, c), grad_std, seed, torch.bfloat16))
    return Ws, Gs
