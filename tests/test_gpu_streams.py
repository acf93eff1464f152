"""Concurrent use: steps on several streams, and from several host threads.

Each (device, stream) pair has its own workspace and status word, and the
kernels carry no state between launches, so steps issued on two streams at
once -- or by two host threads each on its own stream -- must give the same
bits as the same steps run one after the other on one stream.
"""
import threading

import pytest
import torch

import newton_schulz_12_b200 as nsb
from newton_schulz_12_b200 import workloads

pytestmark = pytest.mark.gpu

SHAPES_A = workloads.gpt2_small_shapes(layers=1) + [(130, 68), (300, 1000)]
SHAPES_B = [(512, 2048), (2048, 512), (256, 256), (77, 5)] * 2


class Set:
    def __init__(self, shapes, seed):
        g = torch.Generator(device="cpu").manual_seed(seed)
        self.shapes = shapes
        self.W = [(torch.randn(s, generator=g) * 0.02).cuda() for s in shapes]
        self.M = [torch.zeros(s, device="cuda") for s in shapes]
        self.G = [[(torch.randn(s, generator=g) * 0.01).to(torch.bfloat16).cuda() for s in shapes]
                  for _ in range(3)]

    def clone(self):
        c = Set.__new__(Set)
        c.shapes = self.shapes
        c.W = [w.clone() for w in self.W]
        c.M = [m.clone() for m in self.M]
        c.G = self.G
        return c

    def steps(self, stream=None, n=3):
        for k in range(n):
            nsb.muon_step(self.W, self.G[k], self.M, wd=0.01, stream=stream)


def _same(a, b):
    for x, y in zip(a.W + a.M, b.W + b.M):
        assert torch.equal(x, y)


def test_two_streams_at_once_match_one_stream():
    a, b = Set(SHAPES_A, 1), Set(SHAPES_B, 2)
    a_ref, b_ref = a.clone(), b.clone()
    torch.cuda.synchronize()
    a_ref.steps()
    b_ref.steps()
    torch.cuda.synchronize()
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    for k in range(3):  # interleaved issue: the two streams' launches overlap on the device
        nsb.muon_step(a.W, a.G[k], a.M, wd=0.01, stream=s1)
        nsb.muon_step(b.W, b.G[k], b.M, wd=0.01, stream=s2)
    torch.cuda.synchronize()
    assert nsb.muon_get_status(s1) == 0 and nsb.muon_get_status(s2) == 0
    _same(a, a_ref)
    _same(b, b_ref)


def test_host_threads_each_on_its_own_stream():
    sets = [Set(SHAPES_A, 10 + i) if i % 2 == 0 else Set(SHAPES_B, 10 + i) for i in range(4)]
    refs = [s.clone() for s in sets]
    torch.cuda.synchronize()
    for r in refs:
        r.steps()
    torch.cuda.synchronize()
    errors = []

    def run(s):
        try:
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                s.steps(stream=st)
            st.synchronize()
            if nsb.muon_get_status(st) != 0:
                errors.append(nsb.muon_last_error())
        except Exception as e:  # surfaced below, from the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=run, args=(s,)) for s in sets]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    for s, r in zip(sets, refs):
        _same(s, r)
