"""Pointer validation on a GPU: only device memory of the current device (or
managed memory) reaches a kernel; page-locked host memory, which the device
could read over PCIe, is rejected before anything is launched."""
import ctypes

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_pinned_host_memory_is_rejected():
    import banded_log_domain_b200 as sa

    lib = sa.load()
    B, H, L = 1, 2, 256
    p = sa.make_params(B, H, L, 64, W=8, eps=1.0, T=2, R=2, dtype=torch.bfloat16)
    fws, bws = sa.sinkhorn_attn_workspace_size(p)
    dev = [torch.zeros(B, H, L, 64, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    st = torch.zeros(sa.sinkhorn_attn_state_size(p), device="cuda")
    ws = torch.zeros(max(fws, bws), dtype=torch.uint8, device="cuda")
    pinned = torch.zeros(B, H, L, 64, dtype=torch.bfloat16).pin_memory()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    q, k, v, o = dev
    # the same call with device memory succeeds
    assert lib.sinkhorn_attn_fwd(ctypes.byref(p), P(q), P(k), P(v), None, None, P(o), P(st),
                                 P(ws), ws.numel(), s) == 0
    torch.cuda.synchronize()
    for pos in range(4):
        args = [P(q), P(k), P(v), P(o)]
        args[pos] = P(pinned)
        assert lib.sinkhorn_attn_fwd(ctypes.byref(p), args[0], args[1], args[2], None, None,
                                     args[3], P(st), P(ws), ws.numel(), s) == -1
    pst = torch.zeros(st.numel()).pin_memory()
    assert lib.sinkhorn_attn_fwd(ctypes.byref(p), P(q), P(k), P(v), None, None, P(o), P(pst),
                                 P(ws), ws.numel(), s) == -1
    pmask = torch.ones(B, L, dtype=torch.uint8).pin_memory()
    assert lib.sinkhorn_attn_fwd(ctypes.byref(p), P(q), P(k), P(v), P(pmask), None, P(o), P(st),
                                 P(ws), ws.numel(), s) == -1
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    assert lib.sinkhorn_attn_bwd(ctypes.byref(p), P(q), P(k), P(v), None, None, P(o), P(pinned),
                                 P(st), P(dq), P(dk), P(dv), None, None, P(ws), ws.numel(),
                                 s) == -1
    assert lib.sinkhorn_attn_bwd_static_ws(ctypes.byref(p), P(q), P(k), P(v), None, None, P(o),
                                           P(q), P(st), P(pinned), P(dk), P(dv), None, None,
                                           s) == -1
