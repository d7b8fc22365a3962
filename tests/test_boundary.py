"""The C ABI without a GPU: the library loads, exports every entry point that
include/sinkhorn_attn.h declares, and validates its arguments on the host
before touching the device."""
import ctypes
import os
import re

import pytest
import torch

import banded_log_domain_b200 as sa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sinkhorn_attn.h")


def declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"\b(sinkhorn_attn_\w+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(sa.LIB_PATH)
    names = declared()
    assert len(names) >= 7
    for n in names:
        assert hasattr(lib, n), n
    assert set(sa.EXPORTS) <= set(names)


def P(**kw):
    base = dict(B=2, H=3, L=100, d=64, W=5, eps=0.5, T=4, R=2, dtype=torch.float32)
    base.update(kw)
    B, H, L, d = base.pop("B"), base.pop("H"), base.pop("L"), base.pop("d")
    return sa.make_params(B, H, L, d, **base)


def test_state_and_workspace_sizes():
    assert sa.sinkhorn_attn_state_size(P()) == 2 * 3 * 6 * 100
    assert sa.sinkhorn_attn_state_size(P(R=3, dustbin=True)) == 2 * 3 * 8 * 101
    f, b = sa.sinkhorn_attn_workspace_size(P())
    assert f >= 256 and b >= 256 + 10 * 2 * 3 * 100 * 4
    # O(L): the backward workspace grows linearly in L and not with W
    _, b1 = sa.sinkhorn_attn_workspace_size(P(L=10000, W=5))
    _, b2 = sa.sinkhorn_attn_workspace_size(P(L=10000, W=500))
    _, b3 = sa.sinkhorn_attn_workspace_size(P(L=20000, W=5))
    assert b1 == b2 and 1.9 < b3 / b1 < 2.1


def test_workspace_holds_the_term_block_sum_beyond_four_tail_steps():
    # R <= 4: 2R modifier terms fit one dS sweep; R = 5 adds an fp32 [B][H][L][d]
    # sum of the term blocks plus the per-step vectors
    _, b4 = sa.sinkhorn_attn_workspace_size(P(R=4))
    _, b5 = sa.sinkhorn_attn_workspace_size(P(R=5))
    acc = 2 * 3 * 100 * 64 * 4
    per_step = 8 * 2560  # four [B][H][L] vectors and two term slots per side, 256-aligned
    assert b5 - b4 == acc + per_step
    _, b6 = sa.sinkhorn_attn_workspace_size(P(R=6))
    assert b6 - b5 == per_step


@pytest.mark.parametrize("kw,status", [
    (dict(W=-1), -1), (dict(eps=0.0), -1), (dict(eps=float("nan")), -1), (dict(T=-1), -1),
    (dict(R=-1), -1), (dict(L=-5), -1), (dict(d=32), -2), (dict(R=257), -2),
    (dict(dustbin=True, dustbin_score=float("inf")), -1),
])
def test_invalid_params_rejected(kw, status):
    with pytest.raises(sa.SinkhornAttnError) as e:
        sa.sinkhorn_attn_state_size(P(**kw))
    assert e.value.status == status


def test_bad_enum_and_flags_rejected():
    p = P()
    p.dtype = 7
    assert sa._L().sinkhorn_attn_state_size(ctypes.byref(p), ctypes.byref(ctypes.c_size_t())) == -1
    p = P()
    p.dustbin = 2
    assert sa._L().sinkhorn_attn_state_size(ctypes.byref(p), ctypes.byref(ctypes.c_size_t())) == -1
    p = P()
    p.bwd = 3
    assert sa._L().sinkhorn_attn_state_size(ctypes.byref(p), ctypes.byref(ctypes.c_size_t())) == -1


def test_null_and_host_pointers_rejected_before_launch():
    lib = sa._L()
    p = P()
    ws = ctypes.create_string_buffer(4096)
    buf = ctypes.create_string_buffer(2 * 3 * 100 * 64 * 4 + 64)
    addr = (ctypes.addressof(buf) + 15) & ~15
    # null tensors
    rc = lib.sinkhorn_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None,
                               ctypes.addressof(ws), 4096, None)
    assert rc == -1
    # plain host memory is not a device pointer
    rc = lib.sinkhorn_attn_fwd(ctypes.byref(p), addr, addr, addr, None, None, addr, addr,
                               ctypes.addressof(ws), 4096, None)
    assert rc == -1
    # misaligned
    rc = lib.sinkhorn_attn_fwd(ctypes.byref(p), addr + 4, addr, addr, None, None, addr, addr,
                               ctypes.addressof(ws), 4096, None)
    assert rc == -1


def test_sq_dist_rejects_bad_arguments_on_the_host():
    lib = sa._L()
    buf = ctypes.create_string_buffer(1024)
    addr = (ctypes.addressof(buf) + 15) & ~15
    assert lib.sinkhorn_attn_sq_dist(None, None, -1, sa.SA_F32, None, None) == -1
    assert lib.sinkhorn_attn_sq_dist(None, None, 0, 7, None, None) == -1
    assert lib.sinkhorn_attn_sq_dist(None, None, 0, sa.SA_F32, None, None) == -1  # no output
    # plain host memory is not a device pointer
    assert lib.sinkhorn_attn_sq_dist(addr, addr, 16, sa.SA_BF16, addr, None) == -1


def test_forward_needs_an_iteration():
    # T = R = 0 is rejected before any pointer is looked at (the backward, which
    # does not read T, accepts it)
    lib = sa._L()
    # B = 0: an empty batch is a no-op that succeeds once the parameters pass
    assert lib.sinkhorn_attn_fwd(ctypes.byref(P(B=0, T=1, R=0)), *([None] * 8), 1 << 30, None) == 0
    assert lib.sinkhorn_attn_fwd(ctypes.byref(P(B=0, T=0, R=0)), *([None] * 8), 1 << 30, None) == -1
    p = P(T=0, R=0)
    _, b = sa.sinkhorn_attn_workspace_size(p)
    assert lib.sinkhorn_attn_bwd(ctypes.byref(p), *([None] * 14), b - 1, None) == -3


def test_workspace_too_small():
    lib = sa._L()
    p = P()
    _, b = sa.sinkhorn_attn_workspace_size(p)
    rc = lib.sinkhorn_attn_bwd(ctypes.byref(p), *([None] * 14), b - 1, None)
    assert rc == -3
    rc = lib.sinkhorn_attn_fwd(ctypes.byref(p), *([None] * 8), 16, None)
    assert rc == -3


def test_empty_problem_is_a_noop():
    lib = sa._L()
    p = P(L=0)
    rc = lib.sinkhorn_attn_fwd(ctypes.byref(p), *([None] * 8), 256, None)
    assert rc == 0


def test_strerror_covers_every_status():
    for s in range(0, -9, -1):
        assert sa.strerror(s) and "unknown" not in sa.strerror(s)
    assert "unknown" in sa.strerror(42)


def test_sharded_calls_validate_the_shard_on_the_host():
    lib = sa._L()
    p = P(B=1, H=1, L=50, W=4, dtype=torch.bfloat16)
    noop = sa.EXCHANGE_FN(lambda *a: 0)
    fwd = lambda sh: lib.sinkhorn_attn_fwd_sharded(ctypes.byref(p), sh, *([None] * 7), 1 << 30, None)
    bwd = lambda sh: lib.sinkhorn_attn_bwd_sharded(ctypes.byref(p), sh, *([None] * 11), 1 << 30,
                                                   None)
    for call in (fwd, bwd):
        assert call(None) == -1                                                  # no shard
        assert call(ctypes.byref(sa.sa_shard(4, 4, sa.EXCHANGE_FN(), None))) == -1  # no callback
        assert call(ctypes.byref(sa.sa_shard(30, 30, noop, None))) == -1          # halos overlap
        assert call(ctypes.byref(sa.sa_shard(-1, 0, noop, None))) == -1
    pd = P(B=1, H=1, L=50, W=4, dustbin=True)
    assert lib.sinkhorn_attn_fwd_sharded(ctypes.byref(pd), ctypes.byref(sa.sa_shard(4, 4, noop, None)),
                                         *([None] * 7), 1 << 30, None) == -2      # dustbin


def test_host_step_plans_and_validates_on_the_host():
    lib = sa._L()
    p = P(B=1, H=8, L=100)
    # two slots of the largest group: more groups, smaller workspace
    w1, w4, w8 = (sa.sinkhorn_attn_step_host_workspace_size(p, g) for g in (1, 4, 8))
    assert w1 > w4 > w8 > 0
    with pytest.raises(sa.SinkhornAttnError):
        sa.sinkhorn_attn_step_host_workspace_size(p, 0)
    io = sa.sa_host_step()
    io.groups = 0
    assert lib.sinkhorn_attn_step_host(ctypes.byref(p), ctypes.byref(io), None, 1 << 40, None) == -1
    assert lib.sinkhorn_attn_step_host(ctypes.byref(p), None, None, 1 << 40, None) == -1
    io.groups = 2
    assert lib.sinkhorn_attn_step_host(ctypes.byref(p), ctypes.byref(io), None, 16, None) == -3
    pc = P(B=1, H=8, L=100, check_finite=True)
    assert lib.sinkhorn_attn_step_host(ctypes.byref(pc), ctypes.byref(io), None, 1 << 40, None) == -2
    # host buffers present, but the workspace is not device memory
    buf = torch.zeros(8 * 100 * 64)
    for f in ("q", "k", "v", "dO", "o", "dq", "dk", "dv"):
        setattr(io, f, buf.data_ptr())
    assert lib.sinkhorn_attn_step_host(ctypes.byref(p), ctypes.byref(io), buf.data_ptr(), 1 << 40,
                                       None) == -1


def test_bias_certificate_arithmetic_on_the_host():
    # eta_R = sqrt(sum_t d2 / sum_t n2) over the tensors; R* = smallest R with eta <= tau
    lib = sa._L()
    depths = [4, 0, 2, 1]
    # per depth, three tensors' (d2, n2); ||g_full||^2 = 1 + 2 + 1 = 4 every time
    rows = {0: (0.5, 0.3, 0.2), 1: (1e-6, 0.0, 3e-6), 2: (2e-11, 1e-11, 1e-11), 4: (0.0, 0.0, 0.0)}
    sums = []
    for R in depths:
        for d2, n2 in zip(rows[R], (1.0, 2.0, 1.0)):
            sums += [d2, n2]
    c_d = (ctypes.c_int * 4)(*depths)
    c_s = (ctypes.c_double * len(sums))(*sums)
    eta = (ctypes.c_double * 4)()
    rs = ctypes.c_int(99)
    assert lib.sinkhorn_attn_bias_certificate(4, c_d, 3, c_s, 1e-5, eta, ctypes.byref(rs)) == 0
    want = {0: (1.0 / 4) ** 0.5, 1: (4e-6 / 4) ** 0.5, 2: (4e-11 / 4) ** 0.5, 4: 0.0}
    for i, R in enumerate(depths):
        assert abs(eta[i] - want[R]) <= 1e-15 * max(1.0, want[R])
    assert rs.value == 2  # eta_1 = 1e-3 > tau; eta_2 = 3.2e-6 <= tau; 4 is larger
    assert lib.sinkhorn_attn_bias_certificate(4, c_d, 3, c_s, 1e-12, eta, ctypes.byref(rs)) == 0
    assert rs.value == 4
    assert lib.sinkhorn_attn_bias_certificate(4, c_d, 3, c_s, 0.0, eta, ctypes.byref(rs)) == 0
    assert rs.value == 4  # eta_4 = 0 <= 0
    c_s1 = (ctypes.c_double * 6)(0.0, 0.0, 1e-12, 0.0, 0.0, 0.0)  # ||g_full|| = 0
    c_d1 = (ctypes.c_int * 1)(3)
    assert lib.sinkhorn_attn_bias_certificate(1, c_d1, 3, c_s1, 1.0, eta, ctypes.byref(rs)) == 0
    assert eta[0] == 1e-6 and rs.value == 3
    # invalid arguments
    bad = (ctypes.c_double * 6)(-1.0, 1.0, 0.0, 1.0, 0.0, 1.0)
    assert lib.sinkhorn_attn_bias_certificate(1, c_d1, 3, bad, 1.0, eta, ctypes.byref(rs)) == -1
    assert lib.sinkhorn_attn_bias_certificate(0, c_d, 3, c_s, 1.0, eta, ctypes.byref(rs)) == -1
    assert lib.sinkhorn_attn_bias_certificate(4, c_d, 0, c_s, 1.0, eta, ctypes.byref(rs)) == -1
    assert lib.sinkhorn_attn_bias_certificate(4, c_d, 3, c_s, -1.0, eta, ctypes.byref(rs)) == -1
    assert lib.sinkhorn_attn_bias_certificate(4, c_d, 3, c_s, float("nan"), eta,
                                              ctypes.byref(rs)) == -1
    assert lib.sinkhorn_attn_bias_certificate(4, c_d, 3, None, 1.0, eta, ctypes.byref(rs)) == -1
    neg = (ctypes.c_int * 1)(-2)
    assert lib.sinkhorn_attn_bias_certificate(1, neg, 3, c_s1, 1.0, eta, ctypes.byref(rs)) == -1


def test_binding_does_none_of_the_methods_arithmetic():
    # the score scale and the certificate's eta / R* live in the C library
    src = open(os.path.join(ROOT, "banded_log_domain_b200", "__init__.py")).read()
    assert "score_scale" not in src and "math.sqrt" not in src and "import math" not in src


def test_debug_library_exports_the_same_entry_points():
    # the bounds-checked build (-DSA_DEBUG) is the same C ABI
    assert os.path.exists(sa.DEBUG_LIB_PATH)
    lib = ctypes.CDLL(sa.DEBUG_LIB_PATH)
    for n in declared():
        assert hasattr(lib, n), n
    assert sa.strerror(-8) and "bounds" in sa.strerror(-8)
