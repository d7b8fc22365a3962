"""Banded log-domain Sinkhorn attention on B200 (sm_100a).

A thin ctypes binding over ``libsinkhorn_attn.so`` (C ABI declared in
``include/sinkhorn_attn.h``).  The functions here carry the C entry points'
names and only marshal arguments: they allocate the output, state and
workspace tensors with PyTorch on the inputs' device, pass raw pointers and the
current CUDA stream, and raise on a non-OK status.  Every step of the method
runs in the library's CUDA kernels; there is no fallback of any kind, so a
missing or unloadable library raises on first use.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsinkhorn_attn.so")
# the same library built with device-side bounds checks (-DSA_DEBUG)
DEBUG_LIB_PATH = os.path.join(_PKG, "libsinkhorn_attn_debug.so")
if os.environ.get("SINKHORN_ATTN_DEBUG_LIB") == "1":
    LIB_PATH = DEBUG_LIB_PATH

SA_OK = 0
SA_F32, SA_BF16 = 0, 1
SA_BWD_ONE_REFERENCE, SA_BWD_DIRECT = 0, 1
_STATUS = {0: "SA_OK", -1: "SA_ERR_INVALID_ARG", -2: "SA_ERR_UNSUPPORTED",
           -3: "SA_ERR_WORKSPACE", -4: "SA_ERR_CUDA", -5: "SA_ERR_NONFINITE",
           -6: "SA_ERR_TIMEOUT", -7: "SA_ERR_EXCHANGE", -8: "SA_ERR_BOUNDS"}
SCHEDULES = {"one_reference": SA_BWD_ONE_REFERENCE, "direct": SA_BWD_DIRECT}


class SinkhornAttnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)} ({strerror(status)})")


class sa_params(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int), ("d", ctypes.c_int),
        ("W", ctypes.c_int), ("eps", ctypes.c_float), ("T", ctypes.c_int), ("R", ctypes.c_int),
        ("dtype", ctypes.c_int), ("dustbin", ctypes.c_int), ("dustbin_score", ctypes.c_float),
        ("bwd", ctypes.c_int), ("check_finite", ctypes.c_int),
        ("trace_events", ctypes.c_void_p), ("trace_kinds", ctypes.c_void_p),
        ("trace_count", ctypes.c_void_p), ("trace_cap", ctypes.c_int),
    ]


KERNEL_KINDS = {1: "lse_sweep", 2: "pv", 3: "wsum", 4: "ds", 5: "aux"}

class sa_host_step(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
                ("dO", ctypes.c_void_p), ("mask", ctypes.c_void_p), ("v_dust", ctypes.c_void_p),
                ("o", ctypes.c_void_p), ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p),
                ("dv", ctypes.c_void_p), ("state", ctypes.c_void_p), ("dv_dust", ctypes.c_void_p),
                ("d_dust_score", ctypes.c_void_p), ("groups", ctypes.c_int)]


# int exchange(float* vec, long long row_stride, int rows, void* user, void* stream)
EXCHANGE_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                               ctypes.c_void_p, ctypes.c_void_p)


class sa_shard(ctypes.Structure):
    _fields_ = [("halo_lo", ctypes.c_int), ("halo_hi", ctypes.c_int),
                ("exchange", EXCHANGE_FN), ("user", ctypes.c_void_p)]


class LaunchTrace:
    """CUDA events recorded by the library around each of its kernel launches
    (the ``trace_*`` fields of ``sa_params``).  Pass as ``trace=`` to the
    forward/backward; after synchronising, ``durations()`` lists
    ``(kind, milliseconds)`` per launch."""

    def __init__(self, cap: int = 512):
        self.cap = cap
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * cap)]
        for e in self.events:
            e.record()  # materialise the handle
        self.handles = (ctypes.c_void_p * (2 * cap))(*[e.cuda_event for e in self.events])
        self.kinds = (ctypes.c_int * cap)()
        self.count = ctypes.c_int(0)

    def attach(self, p: "sa_params"):
        p.trace_events = ctypes.cast(self.handles, ctypes.c_void_p)
        p.trace_kinds = ctypes.cast(self.kinds, ctypes.c_void_p)
        p.trace_count = ctypes.cast(ctypes.pointer(self.count), ctypes.c_void_p)
        p.trace_cap = self.cap

    def durations(self):
        n = min(self.count.value, self.cap)
        return [(KERNEL_KINDS.get(self.kinds[i], str(self.kinds[i])),
                 self.events[2 * i].elapsed_time(self.events[2 * i + 1])) for i in range(n)]


_lib = None


def _L():
    """The loaded library; raises if it is missing (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m banded_log_domain_b200.build` "
            "(nvcc, sm_100a); there is no non-CUDA implementation")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(sa_params)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.sinkhorn_attn_state_size.argtypes = [P, ctypes.POINTER(sz)]
    lib.sinkhorn_attn_workspace_size.argtypes = [P, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    lib.sinkhorn_attn_fwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sinkhorn_attn_bwd.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                      sz, vp]
    lib.sinkhorn_attn_bwd_static_ws.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                vp, vp, vp]
    lib.sinkhorn_attn_bwd_static_ws.restype = ctypes.c_int
    lib.sinkhorn_attn_debug_plan.argtypes = [P, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp,
                                             vp, vp, vp]
    lib.sinkhorn_attn_poll.argtypes = [vp, vp]
    lib.sinkhorn_attn_poll_static.argtypes = [vp]
    lib.sinkhorn_attn_bias_certificate.argtypes = [
        ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.c_int, ctypes.POINTER(ctypes.c_double),
        ctypes.c_double, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int)]
    lib.sinkhorn_attn_debug_timeout.argtypes = [vp, ctypes.c_longlong, vp]
    lib.sinkhorn_attn_sq_dist.argtypes = [vp, vp, ctypes.c_longlong, ctypes.c_int, vp, vp]
    lib.sinkhorn_attn_debug_exp2.argtypes = [vp, ctypes.c_longlong, vp, vp, vp]
    lib.sinkhorn_attn_step_host_workspace_size.argtypes = [P, ctypes.c_int, ctypes.POINTER(sz)]
    lib.sinkhorn_attn_step_host.argtypes = [P, ctypes.POINTER(sa_host_step), vp, sz, vp]
    SP = ctypes.POINTER(sa_shard)
    lib.sinkhorn_attn_fwd_sharded.argtypes = [P, SP, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    lib.sinkhorn_attn_bwd_sharded.argtypes = [P, SP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                              sz, vp]
    lib.sinkhorn_attn_strerror.argtypes = [ctypes.c_int]
    lib.sinkhorn_attn_strerror.restype = ctypes.c_char_p
    for f in ("sinkhorn_attn_state_size", "sinkhorn_attn_workspace_size", "sinkhorn_attn_fwd",
              "sinkhorn_attn_bwd", "sinkhorn_attn_debug_plan", "sinkhorn_attn_poll",
              "sinkhorn_attn_poll_static", "sinkhorn_attn_bias_certificate",
              "sinkhorn_attn_debug_exp2",
              "sinkhorn_attn_debug_timeout", "sinkhorn_attn_sq_dist", "sinkhorn_attn_fwd_sharded",
              "sinkhorn_attn_bwd_sharded", "sinkhorn_attn_step_host_workspace_size",
              "sinkhorn_attn_step_host"):
        getattr(lib, f).restype = ctypes.c_int
    _lib = lib
    return lib


def load():
    """Loads the CUDA library now (raises ImportError if it was not built)."""
    return _L()


EXPORTS = ("sinkhorn_attn_state_size", "sinkhorn_attn_workspace_size", "sinkhorn_attn_fwd",
           "sinkhorn_attn_bwd", "sinkhorn_attn_bwd_static_ws", "sinkhorn_attn_debug_plan",
           "sinkhorn_attn_poll", "sinkhorn_attn_poll_static", "sinkhorn_attn_strerror",
           "sinkhorn_attn_debug_timeout", "sinkhorn_attn_bias_certificate",
           "sinkhorn_attn_debug_exp2",
           "sinkhorn_attn_sq_dist", "sinkhorn_attn_fwd_sharded", "sinkhorn_attn_bwd_sharded",
           "sinkhorn_attn_step_host_workspace_size", "sinkhorn_attn_step_host")


def strerror(status: int) -> str:
    return _L().sinkhorn_attn_strerror(int(status)).decode()


def _check(rc: int, what: str):
    if rc != SA_OK:
        raise SinkhornAttnError(rc, what)


def make_params(B, H, L, d, *, W, eps, T, R=2, dtype=torch.float32, dustbin=False,
                dustbin_score=-2.0, schedule="one_reference", check_finite=False) -> sa_params:
    dt = {torch.float32: SA_F32, torch.bfloat16: SA_BF16}[dtype]
    return sa_params(int(B), int(H), int(L), int(d), int(W), float(eps), int(T), int(R), dt,
                     int(bool(dustbin)), float(dustbin_score), SCHEDULES[schedule],
                     int(bool(check_finite)))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _on(device, fn, *args):
    """Calls the C entry point ``fn`` with ``device`` current (the library
    validates every pointer against the current device and launches there)."""
    with torch.cuda.device(device):
        return fn(*args)


def sinkhorn_attn_state_size(p: sa_params) -> int:
    n = ctypes.c_size_t(0)
    _check(_L().sinkhorn_attn_state_size(ctypes.byref(p), ctypes.byref(n)), "state_size")
    return n.value


def sinkhorn_attn_workspace_size(p: sa_params):
    f, b = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(_L().sinkhorn_attn_workspace_size(ctypes.byref(p), ctypes.byref(f), ctypes.byref(b)),
           "workspace_size")
    return f.value, b.value


def _params_for(q, W, eps, T, R, dustbin, dustbin_score, schedule, check_finite):
    B, H, L, d = q.shape
    return make_params(B, H, L, d, W=W, eps=eps, T=T, R=R, dtype=q.dtype, dustbin=dustbin,
                       dustbin_score=dustbin_score, schedule=schedule,
                       check_finite=check_finite)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def sinkhorn_attn_fwd(q, k, v, *, W, eps, T, R=2, mask=None, dustbin=False, dustbin_score=-2.0,
                      v_dust=None, o=None, state=None, ws=None, check_finite=False, trace=None):
    """Forward.  ``q, k, v``: ``[B,H,L,64]`` float32 or bfloat16 CUDA tensors;
    ``mask``: ``[B,L]`` uint8 (1 = valid) or None; ``v_dust``: ``[H,64]`` float32.
    Returns ``(o, state)``; ``state`` is ``[B,H,2R+2,L+dustbin]`` float32."""
    _contig(q, k, v, mask, v_dust, o, state, ws)
    p = _params_for(q, W, eps, T, R, dustbin, dustbin_score, "one_reference", check_finite)
    if trace is not None:
        trace.attach(p)
    dev = q.device
    if o is None:
        o = torch.empty_like(q)
    if state is None:
        state = torch.empty(sinkhorn_attn_state_size(p), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.zeros(sinkhorn_attn_workspace_size(p)[0], dtype=torch.uint8, device=dev)
    rc = _on(dev, _L().sinkhorn_attn_fwd, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(mask),
                                _ptr(v_dust), _ptr(o), _ptr(state), _ptr(ws), ws.numel(),
                                _stream(dev))
    _check(rc, "sinkhorn_attn_fwd")
    B, H, L, _ = q.shape
    return o, state.view(B, H, 2 * R + 2, L + int(bool(dustbin)))


def sinkhorn_attn_bwd(q, k, v, o, dO, state, *, W, eps, R=2, mask=None, dustbin=False,
                      dustbin_score=-2.0, v_dust=None, schedule="one_reference", dq=None, dk=None,
                      dv=None, dv_dust=None, d_dust_score=None, ws=None, check_finite=False,
                      trace=None):
    """Backward of <dO, O> through the tail.  Returns ``(dq, dk, dv, dv_dust)``
    (``dv_dust`` is ``[H,64]`` float32 when ``dustbin``, else None).  With a
    dustbin, a one-element float32 CUDA tensor ``d_dust_score`` receives the
    cotangent of ``dustbin_score`` (summed over batch and heads)."""
    _contig(q, k, v, o, dO, state, mask, v_dust, dq, dk, dv, dv_dust, d_dust_score, ws)
    p = _params_for(q, W, eps, 0, R, dustbin, dustbin_score, schedule, check_finite)
    if trace is not None:
        trace.attach(p)
    dev = q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if dustbin and dv_dust is None:
        dv_dust = torch.empty(q.shape[1], q.shape[3], dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.zeros(sinkhorn_attn_workspace_size(p)[1], dtype=torch.uint8, device=dev)
    rc = _on(dev, _L().sinkhorn_attn_bwd, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(mask),
                                _ptr(v_dust), _ptr(o), _ptr(dO), _ptr(state), _ptr(dq), _ptr(dk),
                                _ptr(dv), _ptr(dv_dust if dustbin else None),
                                _ptr(d_dust_score if dustbin else None), _ptr(ws), ws.numel(),
                                _stream(dev))
    _check(rc, "sinkhorn_attn_bwd")
    return dq, dk, dv, (dv_dust if dustbin else None)


STATIC_SCRATCH_BYTES = 32 << 20


def sinkhorn_attn_bwd_static_ws(q, k, v, o, dO, state, *, W, eps, R=2, mask=None,
                                dustbin=False, dustbin_score=-2.0, v_dust=None,
                                schedule="one_reference", dq=None, dk=None, dv=None,
                                dv_dust=None, d_dust_score=None, trace=None):
    """Backward that takes no workspace: for callers that cannot allocate
    device memory where they run it (see ``sinkhorn_attn_bwd_static_ws`` in
    the C header).  The library's fixed scratch array (``STATIC_SCRATCH_BYTES``
    per GPU) is used instead; calls that overlap on the GPU race.  Pass
    preallocated ``dq, dk, dv`` (and ``dv_dust``) to keep the call free of
    allocations on the Python side too.  ``d_dust_score`` as in
    :func:`sinkhorn_attn_bwd`."""
    _contig(q, k, v, o, dO, state, mask, v_dust, dq, dk, dv, dv_dust, d_dust_score)
    p = _params_for(q, W, eps, 0, R, dustbin, dustbin_score, schedule, False)
    if trace is not None:
        trace.attach(p)
    dev = q.device
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if dustbin and dv_dust is None:
        dv_dust = torch.empty(q.shape[1], q.shape[3], dtype=torch.float32, device=dev)
    rc = _on(dev, _L().sinkhorn_attn_bwd_static_ws, ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(mask),
                                          _ptr(v_dust), _ptr(o), _ptr(dO), _ptr(state), _ptr(dq),
                                          _ptr(dk), _ptr(dv), _ptr(dv_dust if dustbin else None),
                                          _ptr(d_dust_score if dustbin else None), _stream(dev))
    _check(rc, "sinkhorn_attn_bwd_static_ws")
    return dq, dk, dv, (dv_dust if dustbin else None)


def sinkhorn_attn_step_host_workspace_size(p: sa_params, groups: int) -> int:
    n = ctypes.c_size_t()
    _check(_L().sinkhorn_attn_step_host_workspace_size(ctypes.byref(p), int(groups),
                                                       ctypes.byref(n)),
           "sinkhorn_attn_step_host_workspace_size")
    return n.value


def sinkhorn_attn_step_host(q, k, v, dO, *, W, eps, T, R=2, mask=None, dustbin=False,
                            dustbin_score=-2.0, v_dust=None, schedule="one_reference", groups=4,
                            o=None, dq=None, dk=None, dv=None, state=None, dv_dust=None,
                            d_dust_score=None, ws=None, device=None):
    """Forward + backward with inputs and results in host memory: ``q, k, v,
    dO`` are CPU tensors ``[B,H,L,64]`` (page-locked for the copies to overlap
    the compute), ``mask`` ``[B,L]`` uint8 and ``v_dust`` ``[H,64]`` CPU tensors or
    None.  The library copies ``groups`` groups of problems in and results out
    while other groups compute.  Returns CPU tensors ``(o, dq, dk, dv)`` (and
    fills ``state``, ``dv_dust``, ``d_dust_score`` when given); they are final once
    the device's current stream has been synchronised (this function does not
    synchronise).  ``ws``: optional device workspace of
    :func:`sinkhorn_attn_step_host_workspace_size` bytes."""
    for t in (q, k, v, dO, mask, v_dust, o, dq, dk, dv, state, dv_dust, d_dust_score):
        if t is not None and t.is_cuda:
            raise ValueError("sinkhorn_attn_step_host takes host (CPU) tensors")
    _contig(q, k, v, dO, mask, v_dust, o, dq, dk, dv, state, dv_dust, d_dust_score)
    p = _params_for(q, W, eps, T, R, dustbin, dustbin_score, schedule, False)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    pin = q.is_pinned()
    mk = lambda: torch.empty(q.shape, dtype=q.dtype, pin_memory=pin)
    o = mk() if o is None else o
    dq = mk() if dq is None else dq
    dk = mk() if dk is None else dk
    dv = mk() if dv is None else dv
    if ws is None:
        ws = torch.empty(sinkhorn_attn_step_host_workspace_size(p, groups), dtype=torch.uint8,
                         device=dev)
    io = sa_host_step(_ptr(q), _ptr(k), _ptr(v), _ptr(dO), _ptr(mask),
                      _ptr(v_dust if dustbin else None), _ptr(o), _ptr(dq), _ptr(dk), _ptr(dv),
                      _ptr(state), _ptr(dv_dust if dustbin else None),
                      _ptr(d_dust_score if dustbin else None), int(groups))
    rc = _on(dev, _L().sinkhorn_attn_step_host, ctypes.byref(p), ctypes.byref(io), _ptr(ws), ws.numel(),
                                      _stream(dev))
    _check(rc, "sinkhorn_attn_step_host")
    return o, dq, dk, dv


# ---------------------------------------------------------------------------
# sequence sharding (see sa_shard in the C header)
# ---------------------------------------------------------------------------


class _DeviceRows:
    """``rows`` float32 rows of ``L`` entries, ``row_stride`` elements apart,
    at a raw device address, for ``torch.as_tensor``."""

    def __init__(self, ptr, rows, L, row_stride):
        self.__cuda_array_interface__ = {
            "shape": (rows, L), "typestr": "<f4", "data": (int(ptr), False),
            "strides": (int(row_stride) * 4, 4), "version": 3}


def _shard_for(halo_lo, halo_hi, exchange, L, device):
    """The sa_shard of a sharded call: ``exchange(view)`` gets the vector as a
    ``[rows, L]`` float32 tensor view.  Returns (shard, errors, keep-alive)."""
    errors = []

    def cb(ptr, row_stride, rows, user, stream):
        try:
            view = torch.as_tensor(_DeviceRows(ptr, rows, L, row_stride), device=device)
            exchange(view)
            return 0
        except BaseException as e:  # reported by the caller after the C call returns
            errors.append(e)
            return 1

    fn = EXCHANGE_FN(cb)
    return sa_shard(int(halo_lo), int(halo_hi), fn, None), errors, fn


def _check_sharded(rc, what, errors):
    if rc != SA_OK:
        err = SinkhornAttnError(rc, what)
        if errors:
            raise err from errors[0]
        raise err


def sinkhorn_attn_fwd_sharded(q, k, v, *, W, eps, T, R=2, mask=None, halo_lo, halo_hi, exchange,
                              o=None, state=None, ws=None, trace=None):
    """Forward on one shard of a sequence-sharded problem.  ``q, k, v``:
    ``[B,H,L,64]`` for the local sequence (halo tokens included); ``mask``:
    ``[B,L]``; ``exchange(view)`` fills the halo entries of the ``[B*H, L]``
    float32 view from the neighbours (:class:`HaloExchange` over
    torch.distributed).  Returns ``(o, state)`` like :func:`sinkhorn_attn_fwd`;
    only the own tokens' entries are final."""
    _contig(q, k, v, mask, o, state, ws)
    p = _params_for(q, W, eps, T, R, False, -2.0, "one_reference", False)
    if trace is not None:
        trace.attach(p)
    dev = q.device
    B, H, L, _ = q.shape
    o = torch.empty_like(q) if o is None else o
    if state is None:
        state = torch.empty(sinkhorn_attn_state_size(p), dtype=torch.float32, device=dev)
    if ws is None:
        ws = torch.zeros(sinkhorn_attn_workspace_size(p)[0], dtype=torch.uint8, device=dev)
    sh, errors, _keep = _shard_for(halo_lo, halo_hi, exchange, L, dev)
    rc = _on(dev, _L().sinkhorn_attn_fwd_sharded, ctypes.byref(p), ctypes.byref(sh), _ptr(q), _ptr(k),
                                        _ptr(v), _ptr(mask), _ptr(o), _ptr(state), _ptr(ws),
                                        ws.numel(), _stream(dev))
    _check_sharded(rc, "sinkhorn_attn_fwd_sharded", errors)
    return o, state.view(B, H, 2 * R + 2, L)


def sinkhorn_attn_bwd_sharded(q, k, v, o, dO, state, *, W, eps, R=2, mask=None, halo_lo,
                              halo_hi, exchange, schedule="one_reference", dq=None, dk=None,
                              dv=None, ws=None, trace=None):
    """Backward on one shard of a sequence-sharded problem (arguments as in
    :func:`sinkhorn_attn_fwd_sharded` and :func:`sinkhorn_attn_bwd`).  Returns
    ``(dq, dk, dv)``; only the own tokens' rows are final."""
    _contig(q, k, v, o, dO, state, mask, dq, dk, dv, ws)
    p = _params_for(q, W, eps, 0, R, False, -2.0, schedule, False)
    if trace is not None:
        trace.attach(p)
    dev = q.device
    L = q.shape[2]
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    if ws is None:
        ws = torch.zeros(sinkhorn_attn_workspace_size(p)[1], dtype=torch.uint8, device=dev)
    sh, errors, _keep = _shard_for(halo_lo, halo_hi, exchange, L, dev)
    rc = _on(dev, _L().sinkhorn_attn_bwd_sharded, ctypes.byref(p), ctypes.byref(sh), _ptr(q), _ptr(k),
                                        _ptr(v), _ptr(mask), _ptr(o), _ptr(dO), _ptr(state),
                                        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws), ws.numel(),
                                        _stream(dev))
    _check_sharded(rc, "sinkhorn_attn_bwd_sharded", errors)
    return dq, dk, dv


def shard_bounds(L_total, W, rank, world):
    """Contiguous shards of a sequence of ``L_total`` tokens over ``world``
    ranks: ``(own_lo, own_hi, lo, hi)`` with own tokens [own_lo, own_hi) and the
    local sequence [lo, hi) = own tokens plus up to W halo tokens each side.
    Every shard must own at least W tokens."""
    base, extra = divmod(L_total, world)
    own_lo = rank * base + min(rank, extra)
    own_hi = own_lo + base + (1 if rank < extra else 0)
    if world > 1 and base < max(W, 1):
        raise ValueError(f"{L_total} tokens over {world} ranks leave fewer than W = {W} per rank")
    return own_lo, own_hi, max(0, own_lo - W), min(L_total, own_hi + W)


class HaloExchange:
    """The exchange of a sequence-sharded call over torch.distributed (NCCL on
    GPUs, gloo on CPUs): rank r's local vector is [left halo | own | right
    halo]; it sends its first and last own entries (as many as the
    neighbour's halo holds: the halos on the two sides of a boundary are equal,
    W tokens, as ``shard_bounds`` makes them) and receives its halos.  Ranks are
    in sequence order within ``group``."""

    def __init__(self, halo_lo, halo_hi, group=None):
        import torch.distributed as dist

        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        self.halo_lo, self.halo_hi = int(halo_lo), int(halo_hi)
        if (self.halo_lo > 0 and self.rank == 0) or (self.halo_hi > 0 and self.rank == self.world - 1):
            raise ValueError("a halo on a side without a neighbour")

    def _peer(self, r):
        return r if self.group is None else self.dist.get_global_rank(self.group, r)

    def __call__(self, view):
        dist, L = self.dist, view.shape[1]
        hl, hh = self.halo_lo, self.halo_hi
        ops, recvs = [], []
        if hl > 0:
            left = self._peer(self.rank - 1)
            ops.append(dist.P2POp(dist.isend, view[:, hl:2 * hl].contiguous(), left, self.group))
            buf = torch.empty(view.shape[0], hl, dtype=view.dtype, device=view.device)
            ops.append(dist.P2POp(dist.irecv, buf, left, self.group))
            recvs.append((slice(0, hl), buf))
        if hh > 0:
            right = self._peer(self.rank + 1)
            ops.append(dist.P2POp(dist.isend, view[:, L - 2 * hh:L - hh].contiguous(), right,
                                  self.group))
            buf = torch.empty(view.shape[0], hh, dtype=view.dtype, device=view.device)
            ops.append(dist.P2POp(dist.irecv, buf, right, self.group))
            recvs.append((slice(L - hh, L), buf))
        if ops:
            for w in dist.batch_isend_irecv(ops):
                w.wait()
        for sl, buf in recvs:
            view[:, sl].copy_(buf)


def sinkhorn_attn_debug_plan(q, k, state, a, b, *, W, eps, R=2, mask=None, dustbin=False,
                             dustbin_score=-2.0):
    """``P^(a,b)``: ``band [B,H,L,2W+1]``, ``dcol [B,H,L]``, ``drow [B,H,L+1]``
    (the last two only with ``dustbin``)."""
    _contig(q, k, state, mask)
    p = _params_for(q, W, eps, 0, R, dustbin, dustbin_score, "one_reference", False)
    B, H, L, _ = q.shape
    dev = q.device
    band = torch.empty(B, H, L, 2 * W + 1, dtype=torch.float32, device=dev)
    dcol = torch.empty(B, H, L, dtype=torch.float32, device=dev) if dustbin else None
    drow = torch.empty(B, H, L + 1, dtype=torch.float32, device=dev) if dustbin else None
    rc = _on(dev, _L().sinkhorn_attn_debug_plan, ctypes.byref(p), int(a), int(b), _ptr(q), _ptr(k),
                                       _ptr(mask), _ptr(state), _ptr(band), _ptr(dcol),
                                       _ptr(drow), _stream(dev))
    _check(rc, "sinkhorn_attn_debug_plan")
    return band, dcol, drow


def sinkhorn_attn_poll(ws) -> int:
    """Status word recorded in ``ws`` (after synchronising the current stream)."""
    return int(_on(ws.device, _L().sinkhorn_attn_poll, _ptr(ws), _stream(ws.device)))


def sinkhorn_attn_poll_static(device=None) -> int:
    """Status word of the fixed scratch array of :func:`sinkhorn_attn_bwd_static_ws`
    on ``device`` (default: the current one), read and reset after synchronising
    that device's current stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(_on(dev, _L().sinkhorn_attn_poll_static, _stream(dev)))


def sinkhorn_attn_strerror(status: int) -> str:
    return strerror(status)


def sinkhorn_attn_debug_timeout(ws, budget_cycles: int = 1_000_000, device=None) -> int:
    """Runs the library's bounded wait on a barrier nothing completes (test hook
    for the failure path); the timeout lands in the status word of ``ws`` (a
    CUDA tensor of at least 256 bytes) and is read by :func:`sinkhorn_attn_poll`.
    With ``ws=None`` it lands in the static scratch's status word on ``device``
    (read by :func:`sinkhorn_attn_poll_static`)."""
    if ws is not None:
        dev = ws.device
    else:
        dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    return int(_on(dev, _L().sinkhorn_attn_debug_timeout, _ptr(ws), int(budget_cycles),
                   _stream(dev)))


def sinkhorn_attn_debug_exp2(x):
    """``(y_poly, y_mufu)``: 2^x as the row-sum sweeps evaluate it on the FMA pipe
    and on the MUFU unit, for a contiguous float32 CUDA tensor ``x`` (x <= 0)."""
    _contig(x)
    yp, ym = torch.empty_like(x), torch.empty_like(x)
    _check(_on(x.device, _L().sinkhorn_attn_debug_exp2, _ptr(x), x.numel(), _ptr(yp), _ptr(ym),
               _stream(x.device)), "sinkhorn_attn_debug_exp2")
    return yp, ym


def sinkhorn_attn_sq_dist(x, y):
    """``(sum (x - y)^2, sum y^2)`` in double for two contiguous CUDA tensors of
    one shape and dtype (float32 or bfloat16)."""
    _contig(x, y)
    if x.shape != y.shape or x.dtype != y.dtype:
        raise ValueError("x and y must have one shape and dtype")
    dt = {torch.float32: SA_F32, torch.bfloat16: SA_BF16}[x.dtype]
    out = torch.empty(2, dtype=torch.float64, device=x.device)
    _check(_on(x.device, _L().sinkhorn_attn_sq_dist, _ptr(x), _ptr(y), x.numel(), dt, _ptr(out),
               _stream(x.device)), "sinkhorn_attn_sq_dist")
    s = out.cpu()
    return float(s[0]), float(s[1])


def bias_certificate(q, k, v, dO, *, N, Rs=(0, 1, 2, 4), tau=1e-5, W, eps, mask=None,
                     schedule="one_reference"):
    """A-posteriori bias certificate of the stopped base for a solve of N
    iterations (gist.science/de section 3, section 4.1).  For each tail depth R in
    ``Rs`` (0 <= R <= N) the gradients g_R of <dO, O> come from
    :func:`sinkhorn_attn_fwd` / :func:`sinkhorn_attn_bwd` with T = N - R stopped
    iterations; g_full, full backpropagation, from T = 0 and R = N.  Then
    eta_R = ||g_R - g_full|| / ||g_full|| over (dQ, dK, dV), the squared norms from
    :func:`sinkhorn_attn_sq_dist` and eta_R, R* from the C entry point
    ``sinkhorn_attn_bias_certificate``.  Returns ``({R: eta_R}, R*)``, R* the
    smallest R in ``Rs`` with eta_R <= tau (None if none is).  No dustbin."""
    if any(not 0 <= R <= N for R in Rs):
        raise ValueError("every R must lie in [0, N]")

    def grads(T, R):
        o, st = sinkhorn_attn_fwd(q, k, v, W=W, eps=eps, T=T, R=R, mask=mask)
        g = sinkhorn_attn_bwd(q, k, v, o, dO, st, W=W, eps=eps, R=R, mask=mask,
                              schedule=schedule)[:3]
        return g

    full = grads(0, N)
    depths = sorted(set(Rs))
    sums = []
    for R in depths:
        g = full if R == N else grads(N - R, R)
        for a, b in zip(g, full):
            sums.extend(sinkhorn_attn_sq_dist(a, b))
    n = len(depths)
    c_depths = (ctypes.c_int * n)(*depths)
    c_sums = (ctypes.c_double * len(sums))(*sums)
    c_eta = (ctypes.c_double * n)()
    c_rstar = ctypes.c_int(-1)
    _check(_L().sinkhorn_attn_bias_certificate(n, c_depths, len(full), c_sums, float(tau), c_eta,
                                               ctypes.byref(c_rstar)),
           "sinkhorn_attn_bias_certificate")
    eta = {R: float(c_eta[i]) for i, R in enumerate(depths)}
    return eta, (None if c_rstar.value < 0 else int(c_rstar.value))
