"""Muon update (Newton-Schulz orthogonalisation) for B200 / sm_100a.

Thin binding over the C ABI of ``libmuon_b200.so`` (include/muon.h): argument
marshalling only -- every step of the update runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current stream.

The update is the Muon step of the NanoGPT speedrun: orthogonalise each hidden
matrix's Nesterov-momentum update by Newton-Schulz iteration, then apply it
("NanoGPT Speedrun: The Ultimate Guide to Pushing LLM Training Efficiency to Its
Limits", section "Optimizer and Training Strategy Tuning"; "The NanoGPT
speedrun", paragraph "Six records account for most of the speedup", record #3).
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import MUON_BF16, MUON_CAUTIOUS_WD, MUON_FP32, MuonError, check, ptr_array, shape_array

__all__ = [
    "NS_COEFFS", "MuonError", "MuonStepPlan", "MuonNsPlan", "muon_ns_orthogonalize",
    "muon_ns_orthogonalize_schedule",
    "muon_ns_orthogonalize_static", "muon_step", "muon_step_ex", "muon_momentum",
    "muon_apply", "muon_apply_ex", "MUON_CAUTIOUS_WD", "muon_gram_bf16", "muon_poly_bf16", "muon_bx_bf16",
    "muon_bx_apply_bf16", "muon_get_status",
    "muon_last_error", "muon_release", "muon_workspace_bytes", "muon_set_wait_timeout_ms", "muon_set_fault_injection",
    "muon_profile_begin", "muon_profile_end", "muon_version", "MUON_BF16", "MUON_FP32",
]

#: Default quintic coefficients (a, b, c) of X <- aX + (bA + cA^2)X.
NS_COEFFS = (3.4445, -4.7750, 2.0315)


def _stream(stream):
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check_cuda(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _ns_batch(xs):
    """Checks a list of equal-shape bf16 / fp32 CUDA matrices; returns (shape, mode, ptrs)."""
    shape, dtype = tuple(xs[0].shape), xs[0].dtype
    if len(shape) != 2:
        raise ValueError("matrices must be 2-D")
    if dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("matrices must be bf16 or fp32")
    for i, x in enumerate(xs):
        _check_cuda(x, f"xs[{i}]", dtype)
        if tuple(x.shape) != shape:
            raise ValueError("all matrices must have the same shape")
    mode = MUON_BF16 if dtype == torch.bfloat16 else MUON_FP32
    return shape, mode, ptr_array([x.data_ptr() for x in xs])


def muon_ns_orthogonalize(xs, a=NS_COEFFS[0], b=NS_COEFFS[1], c=NS_COEFFS[2], steps=5,
                          stream=None):
    """Orthogonalise every matrix of ``xs`` in place (list of equal-shape CUDA tensors).

    bf16 tensors take the tensor-core path; fp32 tensors take the fp32 SIMT
    verification path.  Returns ``xs``.
    """
    xs = list(xs)
    if not xs:
        return xs
    shape, mode, arr = _ns_batch(xs)
    check(_lib.lib().muon_ns_orthogonalize(len(xs), shape[0], shape[1], arr, a, b, c, steps, mode,
                                           _stream(stream)))
    return xs


def muon_ns_orthogonalize_schedule(xs, schedule, stream=None):
    """``muon_ns_orthogonalize`` with one (a, b, c) triple per step, applied in order."""
    xs = list(xs)
    flat = [float(v) for triple in schedule for v in triple]
    if len(flat) != 3 * len(schedule):
        raise ValueError("schedule must be a sequence of (a, b, c) triples")
    if not xs:
        return xs
    shape, mode, arr = _ns_batch(xs)
    table = (ctypes.c_float * max(1, len(flat)))(*flat)
    check(_lib.lib().muon_ns_orthogonalize_schedule(len(xs), shape[0], shape[1], arr, table,
                                                    len(schedule), mode, _stream(stream)))
    return xs


def muon_ns_orthogonalize_static(xs, a=NS_COEFFS[0], b=NS_COEFFS[1], c=NS_COEFFS[2], steps=5,
                                 status=None, stream=None):
    """muon_ns_orthogonalize for bf16 matrices without any device allocation.

    For callers that may not allocate device memory at the call site (an
    engine that owns all device memory, a fixed memory budget, a loop that
    must not touch an allocator): the library's workspace is a 24 MiB static
    device array instead.  ``status`` is an optional int32 CUDA tensor in which
    a device-side wait timeout is recorded.  Calls that overlap on the GPU
    share that array and must be serialised by the caller.  Returns ``xs``.
    """
    xs = list(xs)
    if not xs:
        return xs
    shape = tuple(xs[0].shape)
    if len(shape) != 2:
        raise ValueError("matrices must be 2-D")
    for i, x in enumerate(xs):
        _check_cuda(x, f"xs[{i}]", torch.bfloat16)
        if tuple(x.shape) != shape:
            raise ValueError("all matrices must have the same shape")
    st = None
    if status is not None:
        _check_cuda(status, "status", torch.int32)
        st = status.data_ptr()
    arr = ptr_array([x.data_ptr() for x in xs])
    check(_lib.lib().muon_ns_orthogonalize_static(len(xs), shape[0], shape[1], arr, a, b, c, steps,
                                                  st, _stream(stream)))
    return xs


def muon_step(params, grads, momentum_bufs, beta=0.95, nesterov=True, lr=0.05, wd=0.0, steps=5,
              stream=None):
    """One Muon step: fp32 ``params`` and ``momentum_bufs`` updated in place from bf16 ``grads``."""
    params, grads, bufs = list(params), list(grads), list(momentum_bufs)
    if not (len(params) == len(grads) == len(bufs)):
        raise ValueError("params, grads and momentum_bufs must have the same length")
    shapes = []
    for i, (w, g, m) in enumerate(zip(params, grads, bufs)):
        _check_cuda(w, f"params[{i}]", torch.float32)
        _check_cuda(g, f"grads[{i}]", torch.bfloat16)
        _check_cuda(m, f"momentum_bufs[{i}]", torch.float32)
        if w.dim() != 2 or w.shape != g.shape or w.shape != m.shape:
            raise ValueError(f"matrix {i}: params, grads and buffers must be equal 2-D shapes")
        shapes.append(tuple(w.shape))
    check(_lib.lib().muon_step(len(params), ptr_array([w.data_ptr() for w in params]),
                               ptr_array([g.data_ptr() for g in grads]),
                               ptr_array([m.data_ptr() for m in bufs]), shape_array(shapes),
                               beta, int(bool(nesterov)), lr, wd, steps, _stream(stream)))


def _step_args(params, grads, momentum_bufs):
    params, grads, bufs = list(params), list(grads), list(momentum_bufs)
    if not (len(params) == len(grads) == len(bufs)):
        raise ValueError("params, grads and momentum_bufs must have the same length")
    shapes = []
    for i, (w, g, m) in enumerate(zip(params, grads, bufs)):
        _check_cuda(w, f"params[{i}]", torch.float32)
        _check_cuda(g, f"grads[{i}]", torch.bfloat16)
        _check_cuda(m, f"momentum_bufs[{i}]", torch.float32)
        if w.dim() != 2 or w.shape != g.shape or w.shape != m.shape:
            raise ValueError(f"matrix {i}: params, grads and buffers must be equal 2-D shapes")
        shapes.append(tuple(w.shape))
    return params, grads, bufs, shapes


def muon_step_ex(params, grads, momentum_bufs, beta=0.95, nesterov=True, lr=0.05, wd=0.0, steps=5,
                 cautious_wd=False, neuron_state=None, beta2=0.95, schedule=None, stream=None):
    """muon_step with per-step coefficients, cautious weight decay and / or
    NorMuon's per-neuron rescale.

    ``schedule``: None (the default triple at every step) or a sequence of
    (a, b, c) triples, one per Newton-Schulz step; it then sets the step count.
    ``neuron_state``: None (off) or a list of fp32 CUDA vectors, one per
    matrix with one entry per row of W (zeros before the first step), updated
    in place.
    """
    params, grads, bufs, shapes = _step_args(params, grads, momentum_bufs)
    table = None
    if schedule is not None:
        flat = [float(v) for triple in schedule for v in triple]
        if len(flat) != 3 * len(schedule):
            raise ValueError("schedule must be a sequence of (a, b, c) triples")
        steps = len(schedule)
        table = (ctypes.c_float * max(1, len(flat)))(*flat)
    state = None
    if neuron_state is not None:
        neuron_state = list(neuron_state)
        if len(neuron_state) != len(params):
            raise ValueError("one neuron_state vector per matrix is required")
        for i, (v, (r, _)) in enumerate(zip(neuron_state, shapes)):
            _check_cuda(v, f"neuron_state[{i}]", torch.float32)
            if v.numel() != r:
                raise ValueError(f"neuron_state[{i}] must hold {r} values (one per row of W)")
        state = ptr_array([v.data_ptr() for v in neuron_state])
    check(_lib.lib().muon_step_ex(len(params), ptr_array([w.data_ptr() for w in params]),
                                  ptr_array([g.data_ptr() for g in grads]),
                                  ptr_array([m.data_ptr() for m in bufs]), shape_array(shapes),
                                  beta, int(bool(nesterov)), lr, wd, steps, table,
                                  MUON_CAUTIOUS_WD if cautious_wd else 0, state, beta2,
                                  _stream(stream)))


class _Replayable:
    """capture / replay for a plan whose call takes a stream."""

    def capture(self, stream=None):
        """Record one call into a CUDA graph (returned; also kept for ``replay``).

        One call runs first on ``stream`` (default: a new side stream) so the
        library's workspace for that stream exists; the next call is only
        recorded (capture does not run it).  Each replay then performs one call,
        launching its kernels without the per-launch host and scheduling gaps.
        The graph bakes in the tensors' addresses, the parameters of this
        moment and that stream's workspace: call ``capture`` again after
        ``update``, and do not call ``muon_release`` or a larger library call on
        that stream while the graph is in use.
        """
        s = stream if isinstance(stream, torch.cuda.Stream) else torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self(s)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            self(s)
        torch.cuda.current_stream().wait_stream(s)
        self._graph = graph
        return graph

    def replay(self):
        """One call by replaying the graph recorded by ``capture`` (on the current stream)."""
        if getattr(self, "_graph", None) is None:
            raise RuntimeError("capture() first")
        self._graph.replay()


class MuonStepPlan(_Replayable):
    """muon_step with its arguments marshalled once, for a fixed set of tensors.

    Checks dtypes, shapes and contiguity at construction; each call then passes
    the cached pointer arrays straight to the C ABI.  The tensors must stay
    alive and keep their storage while the plan is used.  ``capture`` records a
    step in a CUDA graph and ``replay`` runs it (one step per replay).  With
    any of ``cautious_wd``, ``neuron_state`` or ``schedule`` the calls go to
    muon_step_ex (options as there; a schedule fixes the step count).
    """

    def __init__(self, params, grads, momentum_bufs, beta=0.95, nesterov=True, lr=0.05, wd=0.0,
                 steps=5, cautious_wd=False, neuron_state=None, beta2=0.95, schedule=None):
        self.params, self.grads, self.bufs = list(params), list(grads), list(momentum_bufs)
        if not (len(self.params) == len(self.grads) == len(self.bufs)):
            raise ValueError("params, grads and momentum_bufs must have the same length")
        shapes = []
        for i, (w, g, m) in enumerate(zip(self.params, self.grads, self.bufs)):
            _check_cuda(w, f"params[{i}]", torch.float32)
            _check_cuda(g, f"grads[{i}]", torch.bfloat16)
            _check_cuda(m, f"momentum_bufs[{i}]", torch.float32)
            if w.dim() != 2 or w.shape != g.shape or w.shape != m.shape:
                raise ValueError(f"matrix {i}: params, grads and buffers must be equal 2-D shapes")
            shapes.append(tuple(w.shape))
        self.shapes = shapes
        self._p = ptr_array([w.data_ptr() for w in self.params])
        self._g = ptr_array([g.data_ptr() for g in self.grads])
        self._m = ptr_array([m.data_ptr() for m in self.bufs])
        self._s = shape_array(shapes)
        # the refinements (muon_step_ex): per-step triples, cautious decay, NorMuon state
        self._table = None
        if schedule is not None:
            flat = [float(v) for triple in schedule for v in triple]
            if len(flat) != 3 * len(schedule):
                raise ValueError("schedule must be a sequence of (a, b, c) triples")
            steps = len(schedule)
            self._table = (ctypes.c_float * max(1, len(flat)))(*flat)
        self._state = None
        if neuron_state is not None:
            self.neuron_state = list(neuron_state)
            if len(self.neuron_state) != len(self.params):
                raise ValueError("one neuron_state vector per matrix is required")
            for i, (v, (r, _)) in enumerate(zip(self.neuron_state, shapes)):
                _check_cuda(v, f"neuron_state[{i}]", torch.float32)
                if v.numel() != r:
                    raise ValueError(f"neuron_state[{i}] must hold {r} values (one per row of W)")
            self._state = ptr_array([v.data_ptr() for v in self.neuron_state])
        self._ex = (MUON_CAUTIOUS_WD if cautious_wd else 0, float(beta2))
        self._hyper = (float(beta), int(bool(nesterov)), float(lr), float(wd), int(steps))
        self._fn = _lib.lib().muon_step
        self._fn_ex = None
        if self._table is not None or self._state is not None or cautious_wd:
            self._fn_ex = _lib.lib().muon_step_ex

    def update(self, beta=None, nesterov=None, lr=None, wd=None, steps=None):
        """Change hyper-parameters for the following calls (None keeps a value)."""
        if steps is not None and self._table is not None and int(steps) != self._hyper[4]:
            raise ValueError("the step count is fixed by the plan's schedule")
        old = self._hyper
        self._hyper = (float(old[0] if beta is None else beta),
                       int(bool(old[1] if nesterov is None else nesterov)),
                       float(old[2] if lr is None else lr), float(old[3] if wd is None else wd),
                       int(old[4] if steps is None else steps))

    def __call__(self, stream=None):
        beta, nest, lr, wd, steps = self._hyper
        if self._fn_ex is not None:
            flags, beta2 = self._ex
            check(self._fn_ex(len(self.params), self._p, self._g, self._m, self._s, beta, nest, lr,
                              wd, steps, self._table, flags, self._state, beta2, _stream(stream)))
            return
        check(self._fn(len(self.params), self._p, self._g, self._m, self._s, beta, nest, lr, wd,
                       steps, _stream(stream)))

class MuonNsPlan(_Replayable):
    """muon_ns_orthogonalize with its arguments marshalled once, for a fixed
    list of equal-shape matrices (orthogonalised in place by every call).

    For many small matrices the per-call checks and pointer marshalling cost
    about as much host time as the GPU spends on them; the plan pays it once.
    ``capture`` / ``replay`` as for MuonStepPlan.
    """

    def __init__(self, xs, a=NS_COEFFS[0], b=NS_COEFFS[1], c=NS_COEFFS[2], steps=5):
        self.xs = list(xs)
        if not self.xs:
            raise ValueError("no matrices")
        self.shape, self._mode, self._arr = _ns_batch(self.xs)
        self._args = (float(a), float(b), float(c), int(steps))
        self._fn = _lib.lib().muon_ns_orthogonalize

    def __call__(self, stream=None):
        a, b, c, steps = self._args
        check(self._fn(len(self.xs), self.shape[0], self.shape[1], self._arr, a, b, c, steps,
                       self._mode, _stream(stream)))
        return self.xs


def muon_momentum(grads, momentum_bufs, beta=0.95, nesterov=True, sumsq_out=None, stream=None):
    """Momentum stage alone: buffers updated in place; optional per-matrix sum(u^2) (fp32 CUDA)."""
    grads, bufs = list(grads), list(momentum_bufs)
    shapes = []
    for i, (g, m) in enumerate(zip(grads, bufs)):
        _check_cuda(g, f"grads[{i}]", torch.bfloat16)
        _check_cuda(m, f"momentum_bufs[{i}]", torch.float32)
        if g.shape != m.shape or g.dim() != 2:
            raise ValueError(f"matrix {i}: grads and buffers must be equal 2-D shapes")
        shapes.append(tuple(g.shape))
    out = None
    if sumsq_out is not None:
        _check_cuda(sumsq_out, "sumsq_out", torch.float32)
        if sumsq_out.numel() < len(grads):
            raise ValueError("sumsq_out is too small")
        out = sumsq_out.data_ptr()
    check(_lib.lib().muon_momentum(len(grads), ptr_array([g.data_ptr() for g in grads]),
                                   ptr_array([m.data_ptr() for m in bufs]), shape_array(shapes),
                                   beta, int(bool(nesterov)), out, _stream(stream)))


def muon_apply(params, updates, lr=0.05, wd=0.0, stream=None):
    """Apply stage alone: W <- (W - lr*wd*W) - lr*scale*O, fp32, in place."""
    params, updates = list(params), list(updates)
    shapes = []
    for i, (w, o) in enumerate(zip(params, updates)):
        _check_cuda(w, f"params[{i}]", torch.float32)
        _check_cuda(o, f"updates[{i}]", torch.float32)
        if w.shape != o.shape or w.dim() != 2:
            raise ValueError(f"matrix {i}: params and updates must be equal 2-D shapes")
        shapes.append(tuple(w.shape))
    check(_lib.lib().muon_apply(len(params), ptr_array([w.data_ptr() for w in params]),
                                ptr_array([o.data_ptr() for o in updates]), shape_array(shapes),
                                lr, wd, _stream(stream)))


def muon_apply_ex(params, updates, lr=0.05, wd=0.0, cautious_wd=False, row_scale=None, stream=None):
    """muon_apply with cautious decay and / or per-row factors of the update
    (``row_scale``: a list of fp32 CUDA vectors, one entry per row of W)."""
    params, updates = list(params), list(updates)
    shapes = []
    for i, (w, o) in enumerate(zip(params, updates)):
        _check_cuda(w, f"params[{i}]", torch.float32)
        _check_cuda(o, f"updates[{i}]", torch.float32)
        if w.shape != o.shape or w.dim() != 2:
            raise ValueError(f"matrix {i}: params and updates must be equal 2-D shapes")
        shapes.append(tuple(w.shape))
    rs = None
    if row_scale is not None:
        row_scale = list(row_scale)
        for i, (f, (r, _)) in enumerate(zip(row_scale, shapes)):
            _check_cuda(f, f"row_scale[{i}]", torch.float32)
            if f.numel() != r:
                raise ValueError(f"row_scale[{i}] must hold {r} values")
        rs = ptr_array([f.data_ptr() for f in row_scale])
    check(_lib.lib().muon_apply_ex(len(params), ptr_array([w.data_ptr() for w in params]),
                                   ptr_array([o.data_ptr() for o in updates]), shape_array(shapes),
                                   lr, wd, MUON_CAUTIOUS_WD if cautious_wd else 0, rs,
                                   _stream(stream)))


def muon_gram_bf16(X, A=None, stream=None):
    """A = X X^T for a contiguous bf16 batch X (batch, m, k); returns A (batch, m, m)."""
    _check_cuda(X, "X", torch.bfloat16)
    bsz, m, k = X.shape
    if A is None:
        A = torch.empty(bsz, m, m, dtype=torch.bfloat16, device=X.device)
    _check_cuda(A, "A", torch.bfloat16)
    check(_lib.lib().muon_gram_bf16(bsz, m, k, X.data_ptr(), A.data_ptr(), _stream(stream)))
    return A


def muon_poly_bf16(A, b=NS_COEFFS[1], c=NS_COEFFS[2], B=None, stream=None):
    """B = b A + c A A for a contiguous symmetric bf16 batch A (batch, m, m)."""
    _check_cuda(A, "A", torch.bfloat16)
    bsz, m, _ = A.shape
    if B is None:
        B = torch.empty_like(A)
    _check_cuda(B, "B", torch.bfloat16)
    check(_lib.lib().muon_poly_bf16(bsz, m, A.data_ptr(), B.data_ptr(), b, c, _stream(stream)))
    return B


def muon_bx_bf16(B, Xhi, Xlo, a=NS_COEFFS[0], Xhi_out=None, stream=None):
    """X' = a X + B X with X = Xhi + Xlo * 2^(E(Xhi) - 15) (bf16 hi, int8 lo).

    Xlo is overwritten by the int8 part of X'; returns Xhi_out = bf16(X').
    """
    _check_cuda(B, "B", torch.bfloat16)
    _check_cuda(Xhi, "Xhi", torch.bfloat16)
    _check_cuda(Xlo, "Xlo", torch.int8)
    bsz, m, n = Xhi.shape
    if Xhi_out is None:
        Xhi_out = torch.empty_like(Xhi)
    _check_cuda(Xhi_out, "Xhi_out", torch.bfloat16)
    check(_lib.lib().muon_bx_bf16(bsz, m, n, B.data_ptr(), Xhi.data_ptr(), Xlo.data_ptr(),
                                  Xhi_out.data_ptr(), a, _stream(stream)))
    return Xhi_out


def muon_bx_apply_bf16(B, Xhi, Xlo, Ws, n=None, tall=False, a=NS_COEFFS[0], lr=0.05, wd=0.0,
                       cautious=False, stream=None):
    """The last step's X' = a X + B X applied to fp32 weights in the GEMM epilogue.

    ``B`` (batch, m, ldb) bf16, ``Xhi`` (batch, m, ldx) bf16 and ``Xlo``
    (batch, m, ldx) int8 are contiguous batches whose rows may be padded; ``n``
    is X's logical width (default ldx).  ``Ws`` is a list of ``batch`` fp32
    CUDA matrices, each (m, n), or (n, m) with ``tall`` (W = O^T).  Updated in
    place: W <- (W - lr*wd*W) - lr*scale*O (with ``cautious``, the decay only
    where W and O have the same sign).
    """
    _check_cuda(B, "B", torch.bfloat16)
    _check_cuda(Xhi, "Xhi", torch.bfloat16)
    _check_cuda(Xlo, "Xlo", torch.int8)
    bsz, m, ldx = Xhi.shape
    if tuple(Xlo.shape) != (bsz, m, ldx) or B.dim() != 3 or B.shape[0] != bsz or B.shape[1] != m:
        raise ValueError("B must be (batch, m, ldb) and Xlo the shape of Xhi")
    n = ldx if n is None else int(n)
    Ws = list(Ws)
    if len(Ws) != bsz:
        raise ValueError("one weight matrix per batch entry is required")
    want = (n, m) if tall else (m, n)
    for i, w in enumerate(Ws):
        _check_cuda(w, f"Ws[{i}]", torch.float32)
        if tuple(w.shape) != want:
            raise ValueError(f"Ws[{i}] must be {want}, got {tuple(w.shape)}")
    check(_lib.lib().muon_bx_apply_bf16(bsz, m, n, ldx, B.data_ptr(), B.shape[2], Xhi.data_ptr(),
                                        Xlo.data_ptr(), ptr_array([w.data_ptr() for w in Ws]),
                                        int(bool(tall)), a, lr, wd,
                                        MUON_CAUTIOUS_WD if cautious else 0, _stream(stream)))


def muon_get_status(stream=None):
    """Synchronise the stream and return (and clear) its device status word."""
    return _lib.lib().muon_get_status(_stream(stream))


def muon_last_error():
    msg = _lib.lib().muon_last_error()
    return msg.decode() if msg else ""


def muon_release():
    check(_lib.lib().muon_release())


def muon_workspace_bytes(stream=None):
    """Device bytes the library holds for (current device, stream)."""
    out = ctypes.c_longlong(0)
    check(_lib.lib().muon_workspace_bytes(_stream(stream), ctypes.byref(out)))
    return out.value


def muon_set_wait_timeout_ms(ms):
    check(_lib.lib().muon_set_wait_timeout_ms(int(ms)))


def muon_set_fault_injection(mode):
    check(_lib.lib().muon_set_fault_injection(int(mode)))


def muon_profile_begin():
    """Start bracketing every library kernel launch with CUDA events."""
    check(_lib.lib().muon_profile_begin())


def muon_profile_end():
    """Stop timing; returns {kind: (total_ms, launches)} over the recorded launches."""
    k = len(_lib.KERNEL_KINDS)
    ms = (ctypes.c_double * k)()
    n = (ctypes.c_int * k)()
    rc = _lib.lib().muon_profile_end(k, ms, n)
    if rc < 0:
        check(rc)
    return {name: (ms[i], n[i]) for i, name in enumerate(_lib.KERNEL_KINDS)}


def muon_version():
    return _lib.lib().muon_version()
