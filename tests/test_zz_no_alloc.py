"""The allocation-free Newton-Schulz call against the allocating one.

muon_ns_orthogonalize_static serves callers that cannot allocate device memory
where they call the library -- an engine that owns all device memory and
forbids allocation inside its callbacks, a process with a fixed memory budget,
a loop that must never wait on an allocator.  It runs the same kernels on a
static 24 MiB device array instead of an allocated workspace, so its output
must match muon_ns_orthogonalize within the tolerance the other tests use
(relative Frobenius error 3e-2; here it is in fact bit-identical).  Two calls in
a row check that what one call leaves in the shared array does not leak into
the next.  This file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import _lib, workloads

pytestmark = pytest.mark.gpu

TOL = 3e-2


def rel_fro(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def call_static(mats, status):
    """Call the C ABI entry point directly (no Python-side helpers)."""
    arr = _lib.ptr_array([x.data_ptr() for x in mats])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _lib.lib().muon_ns_orthogonalize_static(len(mats), mats[0].shape[0], mats[0].shape[1], arr,
                                                 3.4445, -4.7750, 2.0315, 5, status.data_ptr(),
                                                 stream)
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
        for g, r in zip(got, ref):
            assert rel_fro(g, r) <= TOL
            assert torch.equal(g, r)


def test_static_rejects_oversized_batch():
    x = [torch.zeros(1024, 8192, dtype=torch.bfloat16, device="cuda")]
    arr = _lib.ptr_array([x[0].data_ptr()])
    rc = _lib.lib().muon_ns_orthogonalize_static(1, 1024, 8192, arr, 3.4445, -4.7750, 2.0315, 5,
                                                 None, ctypes.c_void_p(0))
    assert rc == -2
    assert "static scratch" in nsb.muon_last_error()
