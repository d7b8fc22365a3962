"""The host-buffer step (sinkhorn_attn_step_host): inputs and results in host
memory, problems pipelined in groups over the library's copy streams.  Its
results must equal the device-memory calls' on the same inputs: the same
kernels run on each group of (batch, head) problems, which are independent."""
import pytest
import torch

from tests import parity

pytestmark = pytest.mark.gpu

CASES = [
    # (B, H, L, W, T, R, dtype, mask_kind / valid_len, dustbin, groups)
    (1, 6, 1000, 64, 4, 2, "bf16", None, False, 4),       # runs of heads within one batch
    (3, 2, 300, 20, 3, 2, "f32", "holes", False, 2),      # whole batches
    (2, 3, 520, 33, 2, 3, "bf16", (300, 520), False, 5),  # heads, several batches
    (4, 2, 200, 9, 3, 2, "f32", None, True, 3),           # dustbin: whole batches
    (1, 2, 130, 7, 2, 1, "f32", None, False, 1),          # one group
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B{}H{}L{}_{}_db{}_g{}".format(
    c[0], c[1], c[2], c[6], int(c[8]), c[9]))
def test_host_step_equals_device_calls(case):
    import banded_log_domain_b200 as sa

    B, H, L, W, T, R, dtype, mk, db, groups = case
    x = parity.draw_case(B, H, L, dtype=dtype, seed=B * 100 + L,
                         mask_kind=mk if isinstance(mk, str) else None,
                         valid_len=mk if isinstance(mk, tuple) else None, dustbin=db,
                         v_dust_random=db)
    kw = dict(W=W, eps=0.9, R=R, dustbin=db, dustbin_score=-1.1)
    d = parity.to_dev(x)
    o, st = sa.sinkhorn_attn_fwd(d["q"], d["k"], d["v"], T=T, mask=d["mask"], v_dust=d["v_dust"], **kw)
    dsc = torch.zeros(1, device="cuda") if db else None
    g = sa.sinkhorn_attn_bwd(d["q"], d["k"], d["v"], o, d["dO"], st, mask=d["mask"],
                             v_dust=d["v_dust"], d_dust_score=dsc, **kw)
    pin = lambda t: None if t is None else t.contiguous().pin_memory()
    h = {k_: pin(v_) for k_, v_ in x.items()}
    hst = torch.empty(tuple(st.shape), dtype=torch.float32).pin_memory()
    hdvd = torch.empty(H, 64).pin_memory() if db else None
    hdsc = torch.empty(1).pin_memory() if db else None
    out = sa.sinkhorn_attn_step_host(h["q"], h["k"], h["v"], h["dO"], T=T, mask=h["mask"],
                                     v_dust=h["v_dust"], groups=groups, state=hst, dv_dust=hdvd,
                                     d_dust_score=hdsc, **kw)
    torch.cuda.synchronize()
    for name, a, b in zip(("o", "dq", "dk", "dv"), out, (o,) + tuple(g[:3])):
        assert torch.equal(a, b.cpu()), name
    assert torch.equal(hst, st.cpu())
    if db:
        assert torch.allclose(hdvd, g[3].cpu(), rtol=1e-6, atol=1e-7)
        assert torch.allclose(hdsc, dsc.cpu(), rtol=1e-5, atol=1e-7)


def test_host_step_rejects_device_tensors():
    import banded_log_domain_b200 as sa

    q = torch.zeros(1, 1, 8, 64, device="cuda")
    with pytest.raises(ValueError):
        sa.sinkhorn_attn_step_host(q, q, q, q, W=2, eps=1.0, T=1)


@pytest.mark.slow
def test_host_step_long32k_matches_the_oracle():
    """The call bench.py's end-to-end number times, at the full long-context
    size (B=1, H=16, L=32768, W=256, T=20, R=2, bf16) from pinned host buffers,
    against the CPU oracle on two sampled heads (every (batch, head) problem is
    independent)."""
    import numpy as np

    import banded_log_domain_b200 as sa
    import workloads

    w, x = workloads.make("long32k")
    h = {k_: (None if v_ is None else v_.contiguous().pin_memory()) for k_, v_ in x.items()}
    hst = torch.empty(w.B, w.H, 2 * w.R + 2, w.L, dtype=torch.float32).pin_memory()
    o, dq, dk, dv = sa.sinkhorn_attn_step_host(h["q"], h["k"], h["v"], h["dO"], W=w.W, eps=w.eps,
                                               T=w.T, R=w.R, groups=5, state=hst)
    torch.cuda.synchronize()
    heads = [2, 13]
    r = parity.oracle_run(x, W=w.W, eps=w.eps, T=w.T, R=w.R, heads=heads)
    to = lambda t: t.float().double().numpy()
    g = {"o": to(o), "state": hst.double().numpy(),
         "one_reference": (to(dq), to(dk), to(dv), None, None)}
    parity.compare(x, g, r, dtype="bf16", dustbin=False, heads=heads, label="long32k host step")
    assert np.isfinite(g["state"]).all()
