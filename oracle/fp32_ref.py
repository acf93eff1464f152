"""fp32 restatement of the memory-bound Muon steps (test infrastructure only).

The momentum and apply steps are elementwise; their GPU kernels must be
bit-exact against an fp32 computation of the same operation order.  numpy
float32 ufuncs round every multiply and add separately (no fused multiply-add),
so each line below is one correctly rounded IEEE operation, in the order the
kernels perform them:

momentum ([Guide §Optimizer] "Nesterov momentum", lerp reading):
    omb  = fl(1 - beta)
    buf' = fl( fl(beta * buf) + fl(omb * g) )
    u    = fl( fl(omb * g) + fl(beta * buf') )      if nesterov, else buf'

apply ("then scaled and applied"; decoupled weight decay):
    lw   = fl(lr * wd)                  (one scalar per call)
    ls   = fl(lr * scale)               (one scalar per matrix)
    W'   = fl( fl(W - fl(lw * W)) - fl(ls * O) )
    cautious decay: the fl(lw * W) term is 0 where W * O <= 0
    per-neuron factors: O's row r is first fl(O * f_r)

scale (fp32):  s = sqrt(fl(rows / cols)) if rows > cols else 1.

Two more restatements serve the bit-exact check of the last Newton-Schulz
product with the apply fused into it:

pair format (how the bf16 path carries X between steps; defined in the
library's header, not on the pages):
    hi = bf16(X) (nearest even),  E = exponent of hi (hi = 1.f * 2^E),
    q  = nearest-even of (X - hi) / 2^(E-15), clamped to [-128, 127],
    value = hi + q * 2^(E-15)   (q ignored where hi is 0, subnormal or below 2^-111)

fused product:  O = fl(a*x + c)   one rounding of the exact value (an FMA).

[Guide §Optimizer] = "NanoGPT Speedrun: The Ultimate Guide to Pushing LLM
Training Efficiency to Its Limits", section "Optimizer and Training Strategy
Tuning".
"""
from __future__ import annotations

import numpy as np

f32 = np.float32


def momentum_f32(grad, buf, beta, nesterov=True):
    """Return (buf', u) in float32 with the operation order stated above.

    ``grad`` may be bf16 values carried in a float32 array (exact widening).
    """
    g = np.asarray(grad, dtype=f32)
    m = np.asarray(buf, dtype=f32)
    b = f32(beta)
    omb = f32(f32(1.0) - b)
    new_buf = (b * m) + (omb * g)
    if nesterov:
        u = (omb * g) + (b * new_buf)
    else:
        u = new_buf
    assert new_buf.dtype == f32 and u.dtype == f32
    return new_buf, u


def update_scale_f32(rows, cols):
    """fp32 value of sqrt(max(1, rows/cols))."""
    r = f32(f32(rows) / f32(cols))
    return f32(np.sqrt(r)) if r > f32(1.0) else f32(1.0)


def apply_f32(W, O, lr, wd, scale, cautious=False, row_scale=None):
    """W' = (W - lw*W) - ls*O in float32, lw = fl(lr*wd), ls = fl(lr*scale).

    ``cautious``: the lw*W term only where W and O have the same sign (W*O > 0),
    elsewhere W' = W - ls*O.  ``row_scale``: float32 factor per row of W;
    O's row r is fl(O * row_scale[r]) first (the per-neuron rescale).
    """
    W = np.asarray(W, dtype=f32)
    O = np.asarray(O, dtype=f32)
    if row_scale is not None:
        O = O * np.asarray(row_scale, dtype=f32)[:, None]
    lw = f32(f32(lr) * f32(wd))
    ls = f32(f32(lr) * f32(scale))
    decay = lw * W
    if cautious:
        same = ((W > 0) & (O > 0)) | ((W < 0) & (O < 0))
        decay = np.where(same, decay, f32(0.0)).astype(f32)
    out = (W - decay) - (ls * O)
    assert out.dtype == f32
    return out


def bf16_round(x):
    """Round float32 values to the nearest bf16 (ties to even), returned as float32.

    Plain bit arithmetic on the IEEE encoding: keep the top 16 bits after
    adding 0x7FFF plus the lowest kept bit; NaN stays NaN.
    """
    x = np.ascontiguousarray(np.asarray(x, dtype=f32))
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = ((bits + 0x7FFF + lsb) >> 16) << 16
    out = rounded.astype(np.uint32).view(f32)
    nan = np.isnan(x)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


def _bf16_exponent_unit(hi):
    """2^(E-15) for each bf16 value hi (float32 array), 0 where the residual is unused.

    E is hi's binary exponent read from its IEEE encoding (biased exponent field
    minus 127).  The residual is unused when hi is 0 or subnormal (field 0) or
    below 2^-111 (field < 16).
    """
    hi = np.ascontiguousarray(np.asarray(hi, dtype=f32))
    field = (hi.view(np.uint32) >> 23) & 0xFF
    E = field.astype(np.int64) - 127
    unit = np.ldexp(1.0, (E - 15).astype(np.int32))
    return np.where(field >= 16, unit, 0.0)


def pair_value(hi, q):
    """Value of the pair (hi, q) in float64: hi + q * 2^(E-15) (exact; fits fp32)."""
    hi = np.asarray(hi, dtype=f32)
    q = np.asarray(q, dtype=np.int64)
    return hi.astype(np.float64) + q.astype(np.float64) * _bf16_exponent_unit(hi)


def pair_encode(x):
    """The pair (hi, q) of float32 values x: hi as float32 bf16 values, q as int8.

    hi is the nearest-even bf16 of x; q the nearest-even integer of
    (x - hi) / 2^(E-15) clamped to [-128, 127] (0 where the residual is unused).
    x - hi is exact in float64 and the division by a power of two is exact, so
    numpy's rint (ties to even) gives the stated rounding.
    """
    x = np.asarray(x, dtype=f32)
    hi = bf16_round(x)
    unit = _bf16_exponent_unit(hi)
    d = x.astype(np.float64) - hi.astype(np.float64)
    safe = np.where(unit > 0, unit, 1.0)
    q = np.where(unit > 0, np.clip(np.rint(d / safe), -128, 127), 0.0)
    return hi, q.astype(np.int8)


def fma_f32(a, x, c):
    """Correctly rounded float32 of the exact a*x + c (a, x, c float32 values).

    a*x of two float32 values is exact in float64 (at most 48 significant
    bits).  The sum with c is split into s + err exactly (Knuth's two-sum).
    Rounding s to float32 rounds the exact value correctly except when s lies
    exactly halfway between two float32 neighbours and err != 0; then the
    neighbour on err's side is taken.
    """
    a = np.asarray(a, dtype=f32).astype(np.float64)
    x = np.asarray(x, dtype=f32).astype(np.float64)
    c = np.asarray(c, dtype=f32).astype(np.float64)
    p = a * x
    s = p + c
    bp = s - c
    err = (p - bp) + (c - (s - bp))
    r = s.astype(f32)
    other = np.nextafter(r, np.where(s > r.astype(np.float64), f32(np.inf), f32(-np.inf)).astype(f32))
    mid = (r.astype(np.float64) + other.astype(np.float64)) / 2.0
    tie = (err != 0) & (r.astype(np.float64) != s) & (s == mid)
    up = np.maximum(r, other)
    down = np.minimum(r, other)
    fixed = np.where(err > 0, up, down)
    return np.where(tie, fixed, r).astype(f32)
