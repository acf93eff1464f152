"""The allocation-free Newton-Schulz call against the allocating one.

muon_ns_orthogonalize_static serves callers that cannot allocate device memory
where they call the library -- an engine that owns all device memory and
forbids allocation inside its callbacks, a process with a fixed memory budget,
a loop that must never wait on an allocator.  It runs the same kernels on a
static 24 MiB device array instead of an allocated workspace, so its output
must match muon_ns_orthogonalize within the tolerance the other tests use
(relative Frobenius error 3e-2; here it is in fact bit-identical).  Two calls in
a row check that what one call leaves in the shared array does not leak into
the next, and the results are also checked against the fp64 oracle itself.
A call on a fresh stream must leave the library holding no workspace for that
stream (muon_workspace_bytes stays 0), with and without a caller status word.
This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import _lib, workloads
from oracle import muon as oracle

pytestmark = pytest.mark.gpu

TOL = 3e-2


def rel_fro(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def call_static(mats, status, stream=None):
    """Call the C ABI entry point directly (no Python-side helpers)."""
    arr = _lib.ptr_array([x.data_ptr() for x in mats])
    s = stream if stream is not None else torch.cuda.current_stream()
    rc = _lib.lib().muon_ns_orthogonalize_static(len(mats), mats[0].shape[0], mats[0].shape[1], arr,
                                                 3.4445, -4.7750, 2.0315, 5,
                                                 None if status is None else status.data_ptr(),
                                                 ctypes.c_void_p(s.cuda_stream))
    assert rc == 0, nsb.muon_last_error()


@pytest.mark.parametrize("rows,cols,batch", [(768, 3072, 1), (768, 768, 3), (328, 200, 2)])
def test_static_matches_allocating_call_twice(rows, cols, batch):
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        seeds = [7000 + 10 * call + i for i in range(batch)]
        src = [workloads.gaussian((rows, cols), 1.0, seed=s, dtype=torch.bfloat16).cuda()
               for s in seeds]
        ref = [x.clone() for x in src]
        nsb.muon_ns_orthogonalize(ref)
        got = [x.clone() for x in src]
        call_static(got, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        for g, r, x in zip(got, ref, src):
            assert rel_fro(g, r) <= TOL
            assert torch.equal(g, r)
            ora = torch.from_numpy(oracle.newton_schulz(x.double().cpu().numpy()))
            assert rel_fro(g, ora) <= TOL


@pytest.mark.parametrize("with_status", [False, True])
def test_static_on_a_fresh_stream_allocates_nothing(with_status):
    """No workspace appears for the stream the call runs on, twice in a row;
    with no status word the call clears its own slot in the array."""
    stream = torch.cuda.Stream()
    status = torch.zeros(1, dtype=torch.int32, device="cuda") if with_status else None
    for call in range(2):
        src = [workloads.gaussian((328, 200), 1.0, seed=7100 + 10 * call + i, dtype=torch.bfloat16).cuda()
               for i in range(2)]
        got = [x.clone() for x in src]
        torch.cuda.current_stream().synchronize()
        call_static(got, status, stream)
        stream.synchronize()
        assert nsb.muon_workspace_bytes(stream) == 0
        if status is not None:
            assert int(status.item()) == 0
        for g, x in zip(got, src):
            ora = torch.from_numpy(oracle.newton_schulz(x.double().cpu().numpy()))
            assert rel_fro(g, ora) <= TOL


def test_static_rejects_oversized_batch():
    x = [torch.zeros(1024, 8192, dtype=torch.bfloat16, device="cuda")]
    arr = _lib.ptr_array([x[0].data_ptr()])
    rc = _lib.lib().muon_ns_orthogonalize_static(1, 1024, 8192, arr, 3.4445, -4.7750, 2.0315, 5,
                                                 None, ctypes.c_void_p(0))
    assert rc == -2
    assert "static scratch" in nsb.muon_last_error()
