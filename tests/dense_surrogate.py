"""Independent dense float64 implementation of the surrogate, differentiated by
torch autograd.

This is the correctness reference the pages themselves use (Block-Wise
Differentiable Sinkhorn Attention, gist.science/de technical summary section
4.1: the optimised kernel is compared with exact autodiff of the same
surrogate).  It shares nothing with the C oracle: it works on the dense
matrix of the valid tokens (band distance measured in original positions), uses
torch.logsumexp for the sweeps and lets autograd derive the backward, so a
mistake in the oracle's band indexing or in its hand-derived adjoint shows up as
a mismatch.  With ``dustbin`` the augmented problem is built explicitly: one
extra token whose row, column and corner carry the constant dustbin score.
"""
from __future__ import annotations

import math

import torch


def surrogate(q, k, v, *, W, eps, T, R, mask=None, dustbin=False, dustbin_score=-2.0,
              v_dust=None, base=None, stop_base=True):
    """One problem: ``q, k, v`` are ``[L,d]`` float64 (may require grad).

    Returns ``o [L,d]`` and ``state [2R+2, L+db]`` (rows u0, v0, u1, v1, ...),
    with zeros on masked tokens.  ``base``: optional frozen ``[2, L+db]``.
    ``stop_base=False`` lets the gradient run through the T base iterations too
    (full backpropagation through the whole T+R-iteration solve).
    """
    L, d = q.shape
    c = 1.0 / (math.sqrt(d) * eps)
    valid = torch.ones(L, dtype=torch.bool) if mask is None else torch.as_tensor(mask).bool()
    pos = torch.nonzero(valid).flatten()
    n = pos.numel()
    qc, kc, vc = q[pos], k[pos], v[pos]
    S = c * (qc @ kc.T)
    sup = (pos[:, None] - pos[None, :]).abs() <= W
    if dustbin:
        # the score may be a 0-d tensor that requires grad
        sdt = torch.as_tensor(dustbin_score, dtype=q.dtype)
        S = torch.cat([torch.cat([S, sdt.expand(n, 1)], 1), sdt.expand(1, n + 1)], 0)
        sup = torch.cat([torch.cat([sup, torch.ones(n, 1, dtype=torch.bool)], 1),
                         torch.ones(1, n + 1, dtype=torch.bool)], 0)
        vd = torch.zeros(1, d, dtype=q.dtype) if v_dust is None else v_dust.reshape(1, d)
        vc = torch.cat([vc, vd], 0)
    X = S.masked_fill(~sup, float("-inf"))
    m = X.shape[0]

    def row_upd(vv):
        return -torch.logsumexp(X + vv[None, :], dim=1)

    def col_upd(uu):
        return -torch.logsumexp(X + uu[:, None], dim=0)

    full_idx = pos if not dustbin else torch.cat([pos, torch.tensor([L])])
    nst = L + (1 if dustbin else 0)

    def scatter(x):
        out = torch.zeros(nst, dtype=q.dtype)
        return out.index_put((full_idx,), x)

    if base is None:
        with torch.set_grad_enabled(not stop_base and torch.is_grad_enabled()):
            uu = torch.zeros(m, dtype=q.dtype)
            vv = torch.zeros(m, dtype=q.dtype)
            for _ in range(T):
                uu = row_upd(vv)
                vv = col_upd(uu)
    else:
        b = torch.as_tensor(base, dtype=q.dtype)
        uu, vv = b[0][full_idx], b[1][full_idx]
    if stop_base:
        uu, vv = uu.detach(), vv.detach()
    us, vs = [uu], [vv]
    vprev = vv
    for _ in range(R):
        uu = row_upd(vprev)
        vv = col_upd(uu)
        us.append(uu)
        vs.append(vv)
        vprev = vv
    P = torch.exp(X + us[-1][:, None] + vs[-1][None, :])
    oc = P[:n] @ vc
    o = torch.zeros(L, d, dtype=q.dtype).index_put((pos,), oc)
    state = torch.stack([scatter(x) for pair in zip(us, vs) for x in pair])
    return o, state


def surrogate_and_grads(q, k, v, dO, *, v_dust=None, **kw):
    """Forward + autograd VJP of <dO, O> for one problem; all float64 numpy in/out."""
    qt = torch.tensor(q, dtype=torch.float64, requires_grad=True)
    kt = torch.tensor(k, dtype=torch.float64, requires_grad=True)
    vt = torch.tensor(v, dtype=torch.float64, requires_grad=True)
    vdt = None
    if kw.get("dustbin"):
        vd0 = torch.zeros(q.shape[1], dtype=torch.float64) if v_dust is None else \
            torch.tensor(v_dust, dtype=torch.float64)
        vdt = vd0.clone().requires_grad_(True)
    o, st = surrogate(qt, kt, vt, v_dust=vdt, **kw)
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    dvd = None if vdt is None else vdt.grad.numpy()
    return (o.detach().numpy(), st.detach().numpy(), qt.grad.numpy(), kt.grad.numpy(),
            vt.grad.numpy(), dvd)


def dustbin_score_grad(q, k, v, dO, *, dustbin_score, v_dust=None, **kw):
    """d<dO, O> / d(dustbin score) for one problem by autograd (the stopped base
    is a constant, as in the surrogate); float64 numpy in, float out."""
    st = torch.tensor(float(dustbin_score), dtype=torch.float64, requires_grad=True)
    vd = None if v_dust is None else torch.tensor(v_dust, dtype=torch.float64)
    o, _ = surrogate(torch.tensor(q, dtype=torch.float64), torch.tensor(k, dtype=torch.float64),
                     torch.tensor(v, dtype=torch.float64), dustbin=True, dustbin_score=st,
                     v_dust=vd, **kw)
    (o * torch.tensor(dO, dtype=torch.float64)).sum().backward()
    return float(st.grad)
