"""CPU double-precision oracle for banded log-domain Sinkhorn attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the CUDA product path
never does.  The arithmetic lives in ``sinkhorn_oracle.c`` (plain C, double,
OpenMP over rows); this module compiles it with gcc on first use and marshals
numpy arrays through ctypes.  It shares no code with ``banded_log_domain_b200``.

What the oracle computes is stated in the header of ``sinkhorn_oracle.c``
(Block-Wise Differentiable Sinkhorn Attention, gist.science/de technical
summary sections 2.1-2.3).  Every array here is float64; ``[B,H,L,d]`` tensors
are row-major with d contiguous; the mask is ``[B,L]`` uint8 (1 = valid).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sinkhorn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


class _Params(ctypes.Structure):
    _fields_ = [
        ("L", ctypes.c_int),
        ("d", ctypes.c_int),
        ("W", ctypes.c_int),
        ("T", ctypes.c_int),
        ("R", ctypes.c_int),
        ("eps", ctypes.c_double),
        ("dustbin", ctypes.c_int),
        ("dustbin_score", ctypes.c_double),
    ]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (gcc, -O2, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            up = ctypes.POINTER(ctypes.c_ubyte)
            lp = ctypes.POINTER(ctypes.c_longlong)
            pp = ctypes.POINTER(_Params)
            lib.orc_forward.argtypes = [pp, dp, dp, dp, up, dp, dp, dp, dp, lp]
            lib.orc_forward.restype = ctypes.c_int
            lib.orc_backward.argtypes = [pp, ctypes.c_int, dp, dp, dp, up, dp, dp, dp, dp, dp, dp,
                                         dp, dp, lp]
            lib.orc_backward.restype = ctypes.c_int
            lib.orc_plan.argtypes = [pp, ctypes.c_int, ctypes.c_int, dp, dp, up, dp, dp, dp, dp]
            lib.orc_plan.restype = ctypes.c_int
            lib.orc_support_size.argtypes = [pp, up]
            lib.orc_support_size.restype = ctypes.c_longlong
            _lib = lib
    return _lib


def _dp(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _up(a):
    if a is None:
        return None
    assert a.dtype == np.uint8 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_ubyte))


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: exact upcast on the CPU
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _mask(m, B, L):
    if m is None:
        return None
    if hasattr(m, "detach"):
        m = m.detach().to("cpu").numpy()
    m = np.ascontiguousarray(m, dtype=np.uint8)
    assert m.shape == (B, L)
    return m


def _params(L, d, W, T, R, eps, dustbin, dustbin_score):
    return _Params(int(L), int(d), int(W), int(T), int(R), float(eps), int(bool(dustbin)),
                   float(dustbin_score))


def state_len(L, dustbin):
    return L + (1 if dustbin else 0)


def forward(q, k, v, *, W, eps, T, R=2, mask=None, dustbin=False, dustbin_score=-2.0,
            v_dust=None, base=None, count=False):
    """Forward surrogate.  Returns ``(o [B,H,L,d], state [B,H,2R+2,L+db])`` and,
    with ``count=True``, the number of support entries visited per problem.

    ``v_dust``: dustbin value vectors ``[H,d]`` (None = zero).
    ``base``: None for the stopped T-step solve, or ``[B,H,2,L+db]`` holding a
    frozen ``(u0, v0)`` that replaces it.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, L, d = q.shape
    m = _mask(mask, B, L)
    vd = _f64(v_dust)
    bs = _f64(base)
    n = state_len(L, dustbin)
    o = np.zeros((B, H, L, d))
    st = np.zeros((B, H, 2 * R + 2, n))
    visits = np.zeros((B, H), dtype=np.int64)
    p = _params(L, d, W, T, R, eps, dustbin, dustbin_score)
    for b in range(B):
        for h in range(H):
            cnt = ctypes.c_longlong(0)
            rc = lib.orc_forward(
                ctypes.byref(p), _dp(q[b, h]), _dp(k[b, h]), _dp(v[b, h]),
                None if m is None else _up(m[b]),
                None if vd is None else _dp(np.ascontiguousarray(vd[h])),
                None if bs is None else _dp(np.ascontiguousarray(bs[b, h])),
                _dp(o[b, h]), _dp(st[b, h]), ctypes.byref(cnt))
            if rc != 0:
                raise ValueError("oracle forward rejected its arguments")
            visits[b, h] = cnt.value
    return (o, st, visits) if count else (o, st)


def backward(q, k, v, state, dO, *, W, eps, R=2, mask=None, dustbin=False, dustbin_score=-2.0,
             v_dust=None, schedule="direct", count=False, score_grad=False, score_scale=False):
    """Exact surrogate backward.  ``schedule`` is ``"direct"`` (every staircase
    plan by its own exponential) or ``"one_reference"``.  Returns
    ``(dq, dk, dv, dv_dust)``; ``dv_dust`` is ``[H,d]`` summed over the batch.
    With ``score_grad`` a fifth element follows: the cotangent of the dustbin
    score (one scalar shared by every problem, so summed over batch and heads;
    section 2.3 of the gist.science/de summary, one learned dustbin token);
    with ``score_scale`` also a sixth, the sum of |dS| over the dustbin entries
    (the size of what cancels in the fifth: an error scale for comparisons)."""
    lib = _load()
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    st = _f64(state)
    B, H, L, d = q.shape
    m = _mask(mask, B, L)
    vd = _f64(v_dust)
    sched = {"direct": 1, "one_reference": 0}[schedule]
    dq = np.zeros((B, H, L, d))
    dk = np.zeros((B, H, L, d))
    dv = np.zeros((B, H, L, d))
    dvd = np.zeros((H, d))
    visits = np.zeros((B, H), dtype=np.int64)
    dsc = dabs = 0.0
    p = _params(L, d, W, 0, R, eps, dustbin, dustbin_score)
    for b in range(B):
        for h in range(H):
            cnt = ctypes.c_longlong(0)
            part = np.zeros(d)
            gs = np.zeros(2)
            rc = lib.orc_backward(
                ctypes.byref(p), sched, _dp(q[b, h]), _dp(k[b, h]), _dp(v[b, h]),
                None if m is None else _up(m[b]),
                None if vd is None else _dp(np.ascontiguousarray(vd[h])),
                _dp(np.ascontiguousarray(st[b, h])), _dp(dO[b, h]),
                _dp(dq[b, h]), _dp(dk[b, h]), _dp(dv[b, h]), _dp(part), _dp(gs),
                ctypes.byref(cnt))
            if rc != 0:
                raise ValueError("oracle backward rejected its arguments")
            dvd[h] += part
            dsc += float(gs[0])
            dabs += float(gs[1])
            visits[b, h] = cnt.value
    out = (dq, dk, dv, dvd) + ((dsc,) if score_grad else ()) + ((dabs,) if score_scale else ())
    return (out, visits) if count else out


def plan(q, k, state, a, b, *, W, eps, R=2, mask=None, dustbin=False, dustbin_score=-2.0):
    """``P^(a,b)`` on the support.  Returns ``(band [B,H,L,2W+1], dcol [B,H,L],
    drow [B,H,L+1])``; band entry ``t`` of row ``i`` is column ``i-W+t``."""
    lib = _load()
    q, k = _f64(q), _f64(k)
    st = _f64(state)
    B, H, L, d = q.shape
    m = _mask(mask, B, L)
    band = np.zeros((B, H, L, 2 * W + 1))
    dcol = np.zeros((B, H, L + 1))
    drow = np.zeros((B, H, L + 2))
    p = _params(L, d, W, 0, R, eps, dustbin, dustbin_score)
    for bb in range(B):
        for h in range(H):
            rc = lib.orc_plan(ctypes.byref(p), int(a), int(b), _dp(q[bb, h]), _dp(k[bb, h]),
                              None if m is None else _up(m[bb]),
                              _dp(np.ascontiguousarray(st[bb, h])), _dp(band[bb, h]),
                              _dp(dcol[bb, h]), _dp(drow[bb, h]))
            if rc != 0:
                raise ValueError("oracle plan rejected its arguments")
    return band, dcol[..., :L], drow[..., : L + 1]


def support_size(L, W, mask_row=None, dustbin=False):
    """|Omega| (augmented when ``dustbin``) for one sequence."""
    lib = _load()
    p = _params(L, 1, W, 0, 1, 1.0, dustbin, 0.0)
    m = None if mask_row is None else np.ascontiguousarray(mask_row, dtype=np.uint8)
    return int(lib.orc_support_size(ctypes.byref(p), None if m is None else _up(m)))


# ---------------------------------------------------------------------------
# Full backpropagation, the tail-depth-0 gradient and the bias certificate
# (Block-Wise Differentiable Sinkhorn Attention, gist.science/de technical
# summary: section 3 states the a posteriori bias certificate, section 4.1 the
# bias-decay comparison of tail gradients with full backpropagation through time)
# ---------------------------------------------------------------------------

def full_bptt(q, k, v, dO, *, N, W, eps, mask=None, schedule="direct"):
    """Gradients of <dO, O> with backpropagation through the whole N-iteration
    solve (nothing stopped).  The solve from v = 0 is a stopped base of zero
    iterations (a constant) followed by an N-iteration tail, so these are the
    surrogate's exact gradients with T = 0, R = N.  Returns (o, state, (dq, dk, dv))."""
    o, st = forward(q, k, v, W=W, eps=eps, T=0, R=N, mask=mask)
    dq, dk, dv, _ = backward(q, k, v, st, dO, W=W, eps=eps, R=N, mask=mask, schedule=schedule)
    return o, st, (dq, dk, dv)


def stopped_gradients(q, k, v, dO, *, N, W, eps, mask=None):
    """Gradients with every one of the N iterations stopped (tail depth 0):
    O = P V with P = exp(S + u + v) from the stopped duals, so on the support
    dS = P * (dO V^T), dQ = c dS K, dK = c dS^T Q, dV = P^T dO (c = 1/(sqrt(d) eps)).
    Band layout: offset t of row i is column i - W + t.  No dustbin."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    B, H, L, d = q.shape
    c = 1.0 / (np.sqrt(d) * eps)
    _, st = forward(q, k, v, W=W, eps=eps, T=N, R=1, mask=mask)
    P, _, _ = plan(q, k, st, 0, 0, W=W, eps=eps, R=1, mask=mask)  # [B,H,L,2W+1], 0 off the support
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for t in range(2 * W + 1):
        off = t - W  # column j = i + off
        i0, i1 = max(0, -off), min(L, L - off)  # rows whose column is inside [0, L)
        if i1 <= i0:
            continue
        rows = slice(i0, i1)
        cols = slice(i0 + off, i1 + off)
        p = P[:, :, rows, t]                                           # [B,H,n]
        g = np.einsum("bhnd,bhnd->bhn", dO[:, :, rows], v[:, :, cols])  # <dO_i, V_j>
        ds = p * g
        dq[:, :, rows] += c * ds[..., None] * k[:, :, cols]
        dk[:, :, cols] += c * ds[..., None] * q[:, :, rows]
        dv[:, :, cols] += p[..., None] * dO[:, :, rows]
    return dq, dk, dv


def tail_gradients(q, k, v, dO, *, N, R, W, eps, mask=None, schedule="direct"):
    """The surrogate's gradients for a solve of N iterations with tail depth R
    (T = N - R stopped base iterations); R = 0 stops every iteration."""
    if R == 0:
        return stopped_gradients(q, k, v, dO, N=N, W=W, eps=eps, mask=mask)
    _, st = forward(q, k, v, W=W, eps=eps, T=N - R, R=R, mask=mask)
    dq, dk, dv, _ = backward(q, k, v, st, dO, W=W, eps=eps, R=R, mask=mask, schedule=schedule)
    return dq, dk, dv


def bias_certificate(q, k, v, dO, *, N, Rs=(0, 1, 2, 4), tau=1e-5, W, eps, mask=None):
    """For a solve of N iterations, eta_R = ||g_R - g_full|| / ||g_full|| over
    (dQ, dK, dV): the relative size of the gradient that the stopped base omits
    at tail depth R (g_R as in ``tail_gradients``, g_full = ``full_bptt``).
    Returns ({R: eta_R}, R*), R* the smallest R in Rs with eta_R <= tau (None if
    none does)."""
    _, _, gf = full_bptt(q, k, v, dO, N=N, W=W, eps=eps, mask=mask)
    ref = np.sqrt(sum(float(np.sum(x * x)) for x in gf))
    eta = {}
    for R in sorted(Rs):
        g = tail_gradients(q, k, v, dO, N=N, R=R, W=W, eps=eps, mask=mask)
        num = np.sqrt(sum(float(np.sum((a - b) ** 2)) for a, b in zip(g, gf)))
        eta[R] = num / ref if ref > 0 else num
    ok = [R for R in sorted(Rs) if eta[R] <= tau]
    return eta, (ok[0] if ok else None)
