"""Failure detection without a GPU fault.

A host-set flag makes the next tensor-core launch withhold one operand copy in
one CTA, so that CTA's bounded wait runs out: the kernel must record
MUON_ERR_DEVICE_TIMEOUT in the stream's status word, drain what it has in
flight, free its tensor memory and return -- no trap, no hang -- and the
context must stay usable for the next call.  The wait limit is shortened for
the test and restored afterwards.
"""
import numpy as np
import pytest
import torch

import newton_schulz_12_b200 as nsb

pytestmark = pytest.mark.gpu

TIMEOUT = -5


def gram_ref(X):
    Xd = X.double().cpu()
    return Xd @ Xd.transpose(1, 2)


def test_injected_stall_reports_timeout_and_recovers():
    X = (torch.randn(8, 256, 512, generator=torch.Generator().manual_seed(0))).to(torch.bfloat16)
    Xd = X.cuda()
    assert nsb.muon_get_status() == 0
    nsb.muon_set_wait_timeout_ms(200)
    try:
        nsb.muon_set_fault_injection(1)
        nsb.muon_gram_bf16(Xd)
        assert nsb.muon_get_status() == TIMEOUT
        assert "wait" in nsb.muon_last_error()
        assert nsb.muon_get_status() == 0          # read clears the word
    finally:
        nsb.muon_set_fault_injection(0)
        nsb.muon_set_wait_timeout_ms(2000)
    # the next launches run normally on the same context
    A = nsb.muon_gram_bf16(Xd)
    assert nsb.muon_get_status() == 0
    ref = gram_ref(X)
    assert torch.allclose(A.double().cpu(), ref, rtol=2 ** -7, atol=1e-2)
    assert torch.equal(A, A.transpose(1, 2))


def test_injection_flag_is_one_shot():
    X = torch.randn(2, 128, 128).to(torch.bfloat16).cuda()
    nsb.muon_set_wait_timeout_ms(200)
    try:
        nsb.muon_set_fault_injection(1)
        nsb.muon_gram_bf16(X)
        assert nsb.muon_get_status() == TIMEOUT
        nsb.muon_gram_bf16(X)                      # flag consumed: runs clean
        assert nsb.muon_get_status() == 0
    finally:
        nsb.muon_set_fault_injection(0)
        nsb.muon_set_wait_timeout_ms(2000)
