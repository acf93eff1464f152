"""CPU self-test of the block-wise parity bound (tests/blockcheck.py): it must
reject an oracle output with one row, one column or one 128 x 32 epilogue chunk
lost, and accept the same output with bf16-sized noise everywhere."""
import numpy as np
import pytest

from blockcheck import block_errors
from oracle import muon as oracle

TOL = 4 * 3e-2


@pytest.fixture(scope="module")
def ref():
    X = np.random.default_rng(0).standard_normal((256, 768))
    return oracle.newton_schulz(X)


def test_accepts_uniform_noise(ref):
    noisy = ref * (1 + 1e-2 * np.random.default_rng(1).standard_normal(ref.shape))
    assert block_errors(noisy, ref).max() <= TOL


@pytest.mark.parametrize("what", ["row", "col", "chunk", "tall_row"])
def test_rejects_local_loss(ref, what):
    bad = ref.copy()
    r = ref
    if what == "row":
        bad[77, :] = 0.0
    elif what == "col":
        bad[:, 500] = 0.0
    elif what == "chunk":
        bad[128:256, 64:96] = 0.0
    else:
        r = ref.T.copy()
        bad = r.copy()
        bad[400, :] = 0.0
    assert block_errors(bad, r).max() > TOL


def test_ragged_and_thin_shapes():
    for shape in [(1, 17), (17, 1), (1, 32768 // 8), (130, 68)]:
        X = np.random.default_rng(2).standard_normal(shape)
        ref = oracle.newton_schulz(X)
        assert block_errors(ref, ref).max() == 0.0
        bad = ref.copy()
        bad.flat[-1] = -bad.flat[-1] * 3
        assert block_errors(bad, ref).max() > 0.0
