"""Local error bound for the end-to-end parity tests.

The whole-matrix relative Frobenius error can hide a localised mistake: one
lost row of a 768 x 3072 output moves it by only about 3.6 %.  This helper
also bounds the error of every 32 x 32 block against the same block of the
reference, relative to that block's norm, with a floor for blocks whose
reference is near zero (a quarter of the norm the block would have if the
matrix's energy were spread evenly).  A dropped row or column costs a block
at least sqrt(1/32) ~ 18 % of its norm, a dropped epilogue chunk all of it.
"""
import numpy as np

BLOCK = 32
FLOOR = 0.25


def block_errors(got, ref, b=BLOCK, floor=FLOOR):
    """Per-block ||got - ref|| / max(||ref||, floor * even share), as a 2-D array."""
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and ref.ndim == 2
    R, C = ref.shape
    pr, pc = -(-R // b) * b, -(-C // b) * b

    def blocksum(x):
        p = np.zeros((pr, pc))
        p[:R, :C] = x
        return p.reshape(pr // b, b, pc // b, b).sum(axis=(1, 3))

    err = np.sqrt(blocksum((got - ref) ** 2))
    nrm = np.sqrt(blocksum(ref ** 2))
    cnt = blocksum(np.ones_like(ref))
    rms = np.linalg.norm(ref) / np.sqrt(R * C)
    den = np.maximum(nrm, floor * rms * np.sqrt(cnt))
    den = np.where(den > 0, den, 1.0)
    return err / den


def assert_blocks(got, ref, tol, what=""):
    e = block_errors(got, ref)
    worst = np.unravel_index(int(np.argmax(e)), e.shape)
    assert e.max() <= tol, (f"{what}: block {worst} (rows {worst[0] * BLOCK}.., cols {worst[1] * BLOCK}..) "
                            f"has relative error {e.max():.3e} > {tol}")
