"""Shared machinery of the GPU-vs-oracle parity tests.

Tolerances (the stated contract of this library):
  * duals and plans: absolute 1e-5 over valid entries, for both storage types
    (the duals are float32 in both; with bf16 storage only Q, K, V, dO and the
    outputs are rounded);
  * O, dQ, dK, dV, dv_dust: relative l2 (||x - y|| / ||y|| over the compared
    elements) 1e-4 for fp32 storage, 2e-2 for bf16 storage (the outputs are
    rounded to bf16, whose unit roundoff is 2^-8);
  * the dustbin score's cotangent (a scalar): the larger of the relative bound
    above and SCORE_ROUND times sum |dS_e|, the total size of the
    dustbin-entry cotangents it sums; they cancel down to a remainder 10^3 to
    10^4 times smaller on these random inputs, so its error follows their size;
  * the support (which plan entries are non-zero) and the zeros of masked
    tokens: exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

DUAL_ATOL = {"f32": 1e-5, "bf16": 1e-5}
REL_L2 = {"f32": 1e-4, "bf16": 2e-2}
# relative accuracy of the inputs of the dustbin-entry cotangents: fp32 duals
# and vector cotangents (about 1e-6); with bf16 storage the row dot <dO, O>
# reads O rounded to 2^-9, averaged over 64 dimensions
SCORE_ROUND = {"f32": 2.0 ** -20, "bf16": 2.0 ** -12}


def rel_l2(x, y):
    x = np.asarray(x, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    den = np.linalg.norm(y.ravel())
    num = np.linalg.norm((x - y).ravel())
    return num / den if den > 0 else num


def to_dev(x, dev="cuda"):
    return {k: (None if v is None else v.to(dev)) for k, v in x.items()}


def gpu_run(x, *, W, eps, T, R, dustbin=False, dustbin_score=-2.0, schedules=("one_reference",),
            plans=()):
    """Forward + backward(s) through the C ABI.  Returns numpy float64 arrays."""
    import banded_log_domain_b200 as sa

    d = to_dev(x)
    o, st = sa.sinkhorn_attn_fwd(d["q"], d["k"], d["v"], W=W, eps=eps, T=T, R=R, mask=d["mask"],
                                 dustbin=dustbin, dustbin_score=dustbin_score,
                                 v_dust=d["v_dust"])
    out = {"o": o, "state": st}
    for s in schedules:
        dsc = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda") if dustbin else None
        dq, dk, dv, dvd = sa.sinkhorn_attn_bwd(d["q"], d["k"], d["v"], o, d["dO"], st, W=W,
                                               eps=eps, R=R, mask=d["mask"], dustbin=dustbin,
                                               dustbin_score=dustbin_score, v_dust=d["v_dust"],
                                               schedule=s, d_dust_score=dsc)
        out[s] = (dq, dk, dv, dvd, dsc)
    for (a, b) in plans:
        out[("plan", a, b)] = sa.sinkhorn_attn_debug_plan(d["q"], d["k"], st, a, b, W=W, eps=eps,
                                                          R=R, mask=d["mask"], dustbin=dustbin,
                                                          dustbin_score=dustbin_score)
    torch.cuda.synchronize()

    def np_(t):
        if t is None:
            return None
        if isinstance(t, tuple):
            return tuple(np_(u) for u in t)
        return t.detach().float().cpu().double().numpy()

    return {k: np_(v) for k, v in out.items()}


def oracle_run(x, *, W, eps, T, R, dustbin=False, dustbin_score=-2.0, plans=(), heads=None):
    """The oracle on the same inputs (optionally a subset of heads)."""
    sel = (slice(None), heads if heads is not None else slice(None))
    q, k, v, dO = (x[n][sel] for n in ("q", "k", "v", "dO"))
    vd = x["v_dust"]
    if vd is not None and heads is not None:
        vd = vd[heads]
    kw = dict(W=W, eps=eps, R=R, mask=x["mask"], dustbin=dustbin, dustbin_score=dustbin_score)
    o, st = oracle.forward(q, k, v, T=T, v_dust=vd, **kw)
    g = oracle.backward(q, k, v, st, dO, v_dust=vd, schedule="direct", score_grad=True,
                        score_scale=True, **kw)
    out = {"o": o, "state": st, "grads": g}
    for (a, b) in plans:
        out[("plan", a, b)] = oracle.plan(q, k, st, a, b, **kw)
    return out


def valid_mask(x, B, L):
    m = x["mask"]
    return np.ones((B, L), bool) if m is None else m.numpy().astype(bool)


def compare(x, g, r, *, dtype, dustbin, schedules=("one_reference",), heads=None, rows=None,
            label=""):
    """Asserts parity of GPU results ``g`` with oracle results ``r``.

    ``heads``: the head indices the oracle ran on; ``rows``: optional token
    slice restricting the comparison (for windowed oracle runs)."""
    B, H, L, d = x["q"].shape
    hs = list(range(H)) if heads is None else list(heads)
    rs = slice(None) if rows is None else rows
    vm = valid_mask(x, B, L)[:, rs]
    tol = REL_L2[dtype]
    # duals over valid entries (and the dustbin slot)
    gs = g["state"][:, hs]
    rsd = r["state"]
    gs_t, rs_t = gs[..., :L][..., rs], rsd[..., :L][..., rs]
    m = np.broadcast_to(vm[:, None, None, :], gs_t.shape)
    err = np.abs(gs_t - rs_t)[m].max() if m.any() else 0.0
    assert err <= DUAL_ATOL[dtype], f"{label} duals max abs err {err}"
    assert np.all(gs_t[~m] == 0), f"{label} masked duals not zero"
    if dustbin and rows is None:
        e2 = np.abs(gs[..., L] - rsd[..., L]).max()
        assert e2 <= DUAL_ATOL[dtype], f"{label} dustbin duals err {e2}"
    # O
    go = g["o"][:, hs][:, :, rs]
    ro = r["o"][:, :, rs]
    mo = np.broadcast_to(vm[:, None, :, None], go.shape)
    e = rel_l2(go[mo], ro[mo])
    assert e <= tol, f"{label} O rel-l2 {e}"
    assert np.all(go[~mo] == 0), f"{label} masked O not zero"
    rdq, rdk, rdv, rdvd, rdsc, rdabs = r["grads"]
    for s in schedules:
        gdq, gdk, gdv, gdvd, gdsc = g[s]
        for name, gt, rt in (("dQ", gdq, rdq), ("dK", gdk, rdk), ("dV", gdv, rdv)):
            gt = gt[:, hs][:, :, rs]
            rt = rt[:, :, rs]
            e = rel_l2(gt[mo], rt[mo])
            assert e <= tol, f"{label} {s} {name} rel-l2 {e}"
            assert np.all(gt[~mo] == 0), f"{label} {s} masked {name} not zero"
        if dustbin and rows is None and heads is None:
            e = rel_l2(gdvd, rdvd)
            assert e <= max(tol, 1e-4) or np.abs(rdvd).max() == 0, f"{label} dv_dust rel-l2 {e}"
            # the dustbin score's cotangent: one scalar summed over every problem,
            # the small remainder of dustbin-entry cotangents that cancel, so its
            # error scales with their total size sum |dS_e| (with bf16 storage
            # the row dot <dO, O> also reads the rounded O)
            gs, rs_ = float(gdsc[0]), float(rdsc)
            bound = max(tol * abs(rs_), SCORE_ROUND[dtype] * rdabs)
            assert abs(gs - rs_) <= bound, f"{label} {s} d_score {gs} vs {rs_} (bound {bound})"


def compare_plans(g, r, plans, *, dtype="f32", heads=None, label=""):
    for key in plans:
        gb, gdc, gdr = g[("plan",) + tuple(key)]
        rb, rdc, rdr = r[("plan",) + tuple(key)]
        if heads is not None:
            gb = gb[:, heads]
            gdc = None if gdc is None else gdc[:, heads]
            gdr = None if gdr is None else gdr[:, heads]
        # support bit-exact, values within the dual tolerance
        assert np.array_equal(gb != 0, rb != 0), f"{label} plan {key} support differs"
        e = np.abs(gb - rb).max()
        assert e <= DUAL_ATOL[dtype], f"{label} plan {key} max abs err {e}"
        if gdc is not None:
            assert np.abs(gdc - rdc).max() <= DUAL_ATOL[dtype]
            assert np.abs(gdr - rdr).max() <= DUAL_ATOL[dtype]


def draw_case(B, H, L, *, dtype="f32", seed=0, mask_kind=None, valid_len=None, dustbin=False,
              v_dust_random=False):
    x = workloads.draw(B, H, L, 64, dtype=dtype, seed=seed, valid_len=valid_len,
                       mask_kind=mask_kind, dustbin=dustbin)
    if dustbin and v_dust_random:
        g = torch.Generator().manual_seed(seed + 1)
        x["v_dust"] = torch.randn(H, 64, generator=g)
    return x
