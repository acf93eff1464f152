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

scale (fp32):  s = sqrt(fl(rows / cols)) if rows > cols else 1.

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


def apply_f32(W, O, lr, wd, scale):
    """W' = (W - lw*W) - ls*O in float32, lw = fl(lr*wd), ls = fl(lr*scale)."""
    W = np.asarray(W, dtype=f32)
    O = np.asarray(O, dtype=f32)
    lw = f32(f32(lr) * f32(wd))
    ls = f32(f32(lr) * f32(scale))
    out = (W - (lw * W)) - (ls * O)
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
