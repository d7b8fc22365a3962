"""The backward entry point that takes no workspace (sinkhorn_attn_bwd_static_ws).

It serves callers that cannot allocate device memory where they run the
backward (a host framework that owns all device memory, latency-critical code
that cannot take cudaMalloc's synchronisation) and have no buffer to lend.  It
must give the same results as sinkhorn_attn_bwd, call after call, although its
scratch array is shared and keeps the previous call's contents.  This file is
collected last on purpose.
"""
import numpy as np
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu


def _problem(seed, B, H, L, W, dtype, dustbin):
    x = parity.draw_case(B, H, L, dtype=dtype, seed=seed, valid_len=(L // 2, L),
                         dustbin=dustbin, v_dust_random=dustbin)
    return {k: (None if v is None else v.cuda()) for k, v in x.items()}


def test_static_scratch_backward_matches_workspace_backward():
    import banded_log_domain_b200 as sa

    cases = [
        # two different problems in a row: the second must not see the first's scratch
        dict(seed=3, B=2, H=3, L=700, W=40, eps=0.7, T=5, dtype="f32", dustbin=True),
        dict(seed=4, B=1, H=2, L=333, W=17, eps=1.0, T=3, dtype="bf16", dustbin=False),
    ]
    for c in cases:
        x = _problem(c["seed"], c["B"], c["H"], c["L"], c["W"], c["dtype"], c["dustbin"])
        kw = dict(W=c["W"], eps=c["eps"], R=2, mask=x["mask"], dustbin=c["dustbin"],
                  dustbin_score=-1.5, v_dust=x["v_dust"])
        o, st = sa.sinkhorn_attn_fwd(x["q"], x["k"], x["v"], T=c["T"], **kw)
        for sched in ("one_reference", "direct"):
            ref = sa.sinkhorn_attn_bwd(x["q"], x["k"], x["v"], o, x["dO"], st, schedule=sched,
                                       **kw)
            out = [torch.empty_like(x["q"]) for _ in range(3)]
            dvd = torch.empty(c["H"], 64, device="cuda") if c["dustbin"] else None
            got = sa.sinkhorn_attn_bwd_static_ws(x["q"], x["k"], x["v"], o, x["dO"], st,
                                                 schedule=sched, dq=out[0], dk=out[1], dv=out[2],
                                                 dv_dust=dvd, **kw)
            torch.cuda.synchronize()
            tol = parity.REL_L2[c["dtype"]]
            for a, b in zip(got, ref):
                if b is None:
                    continue
                a = a.double().cpu().numpy()
                b = b.double().cpu().numpy()
                assert parity.rel_l2(a, b) <= tol
                assert np.array_equal(a == 0, b == 0)


def test_static_scratch_rejects_oversize_problem():
    import banded_log_domain_b200 as sa

    p = sa.make_params(1, 16, 32768, 64, W=256, eps=1.0, T=20, R=2, dtype=torch.bfloat16)
    assert sa.sinkhorn_attn_workspace_size(p)[1] > sa.STATIC_SCRATCH_BYTES
    q = torch.zeros(1, 16, 32768, 64, dtype=torch.bfloat16, device="cuda")
    st = torch.zeros(1, 16, 6, 32768, device="cuda")
    with pytest.raises(sa.SinkhornAttnError) as e:
        sa.sinkhorn_attn_bwd_static_ws(q, q, q, q, q, st, W=256, eps=1.0, R=2)
    assert e.value.status == -3
