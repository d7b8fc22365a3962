"""The backward entry point that takes no workspace (sinkhorn_attn_bwd_static_ws).

It serves callers that cannot allocate device memory where they run the
backward (a host framework that owns all device memory, latency-critical code
that cannot take cudaMalloc's synchronisation) and have no buffer to lend.  It
must give the same results as sinkhorn_attn_bwd, call after call, although its
scratch array is shared and keeps the previous call's contents; a condition a
call records there (a bounded wait that gave up) must reach the caller through
sinkhorn_attn_poll_static.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu

SA_ERR_TIMEOUT = -6


def _problem(seed, B, H, L, W, dtype, dustbin):
    x = parity.draw_case(B, H, L, dtype=dtype, seed=seed, valid_len=(L // 2, L),
                         dustbin=dustbin, v_dust_random=dustbin)
    return x, {k: (None if v is None else v.cuda()) for k, v in x.items()}


def _static_vs_workspace(sa, x, c, kw):
    """Both schedules of the static-scratch backward against the workspace backward."""
    o, st = sa.sinkhorn_attn_fwd(x["q"], x["k"], x["v"], T=c["T"], **kw)
    for sched in ("one_reference", "direct"):
        dsc_ref = torch.full((1,), float("nan"), device="cuda") if c["dustbin"] else None
        ref = sa.sinkhorn_attn_bwd(x["q"], x["k"], x["v"], o, x["dO"], st, schedule=sched,
                                   d_dust_score=dsc_ref, **kw)
        out = [torch.empty_like(x["q"]) for _ in range(3)]
        dvd = torch.empty(c["H"], 64, device="cuda") if c["dustbin"] else None
        dsc = torch.full((1,), float("nan"), device="cuda") if c["dustbin"] else None
        got = sa.sinkhorn_attn_bwd_static_ws(x["q"], x["k"], x["v"], o, x["dO"], st,
                                             schedule=sched, dq=out[0], dk=out[1], dv=out[2],
                                             dv_dust=dvd, d_dust_score=dsc, **kw)
        torch.cuda.synchronize()
        tol = parity.REL_L2[c["dtype"]]
        for a, b in zip(got, ref):
            if b is None:
                continue
            a = a.double().cpu().numpy()
            b = b.double().cpu().numpy()
            assert parity.rel_l2(a, b) <= tol
            assert np.array_equal(a == 0, b == 0)
        if c["dustbin"]:
            g, r = float(dsc.item()), float(dsc_ref.item())
            assert np.isfinite(g) and abs(g - r) <= 1e-5 * max(1.0, abs(r)), (g, r)
    return o, st


def test_static_scratch_backward_matches_workspace_backward():
    import banded_log_domain_b200 as sa

    cases = [
        # two different problems in a row: the second must not see the first's scratch
        dict(seed=3, B=2, H=3, L=700, W=40, eps=0.7, T=5, dtype="f32", dustbin=True),
        dict(seed=4, B=1, H=2, L=333, W=17, eps=1.0, T=3, dtype="bf16", dustbin=False),
    ]
    for c in cases:
        _, x = _problem(c["seed"], c["B"], c["H"], c["L"], c["W"], c["dtype"], c["dustbin"])
        kw = dict(W=c["W"], eps=c["eps"], R=2, mask=x["mask"], dustbin=c["dustbin"],
                  dustbin_score=-1.5, v_dust=x["v_dust"])
        _static_vs_workspace(sa, x, c, kw)
    assert sa.sinkhorn_attn_poll_static() == 0


def test_static_scratch_backward_matches_the_oracle():
    """The tensor-core (bf16) path of the static-scratch backward against the
    CPU oracle directly, at the library's stated tolerances."""
    import banded_log_domain_b200 as sa

    x, d = _problem(9, 1, 2, 600, 48, "bf16", False)
    kw = dict(W=48, eps=0.9, T=4, R=2)
    o, st = sa.sinkhorn_attn_fwd(d["q"], d["k"], d["v"], mask=d["mask"], **kw)
    kwb = dict(kw)
    kwb.pop("T")
    dq, dk, dv, _ = sa.sinkhorn_attn_bwd_static_ws(d["q"], d["k"], d["v"], o, d["dO"], st,
                                                  mask=d["mask"], **kwb)
    torch.cuda.synchronize()
    r = parity.oracle_run(x, **kw)
    g = {"o": o.double().cpu().numpy(), "state": st.double().cpu().numpy(),
         "one_reference": tuple(t.double().cpu().numpy() for t in (dq, dk, dv)) + (None, None)}
    parity.compare(x, g, r, dtype="bf16", dustbin=False, label="static scratch vs oracle")
    assert sa.sinkhorn_attn_poll_static() == 0


def test_static_scratch_rejects_oversize_problem_then_runs_in_size():
    import banded_log_domain_b200 as sa

    p = sa.make_params(1, 16, 32768, 64, W=256, eps=1.0, T=20, R=2, dtype=torch.bfloat16)
    assert sa.sinkhorn_attn_workspace_size(p)[1] > sa.STATIC_SCRATCH_BYTES
    q = torch.zeros(1, 16, 32768, 64, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, 16, 6, 32768, device="cuda")
    with pytest.raises(sa.SinkhornAttnError) as e:
        sa.sinkhorn_attn_bwd_static_ws(q, q, q, q, q, st, W=256, eps=1.0, R=2)
    assert e.value.status == -3
    del q, st
    # the rejection leaves nothing behind: an in-size call right after matches
    c = dict(seed=5, B=1, H=2, L=400, W=30, eps=0.8, T=3, dtype="bf16", dustbin=False)
    _, x = _problem(c["seed"], c["B"], c["H"], c["L"], c["W"], c["dtype"], c["dustbin"])
    kw = dict(W=c["W"], eps=c["eps"], R=2, mask=x["mask"])
    _static_vs_workspace(sa, x, c, kw)
    assert sa.sinkhorn_attn_poll_static() == 0


def test_static_scratch_reports_a_timeout():
    """A bounded wait that gives up on the static scratch's status word reaches
    the caller through sinkhorn_attn_poll_static, which then resets it; a
    backward call in between does not clear it."""
    import banded_log_domain_b200 as sa

    assert sa.sinkhorn_attn_poll_static() == 0
    assert sa.sinkhorn_attn_debug_timeout(None, 200_000) == 0
    c = dict(seed=6, B=1, H=1, L=256, W=12, eps=1.0, T=2, dtype="bf16", dustbin=False)
    _, x = _problem(c["seed"], c["B"], c["H"], c["L"], c["W"], c["dtype"], c["dustbin"])
    kw = dict(W=c["W"], eps=c["eps"], R=2, mask=x["mask"])
    _static_vs_workspace(sa, x, c, kw)
    assert sa.sinkhorn_attn_poll_static() == SA_ERR_TIMEOUT
    assert sa.sinkhorn_attn_poll_static() == 0
