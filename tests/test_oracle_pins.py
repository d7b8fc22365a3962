"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

No page prints a worked example, so each pin is a closed form, an invariant, a
special case that reduces to a library routine, an independent implementation
(dense autograd), or finite differences.  Together they are chosen so that a
plausible slip in the oracle (a wrong axis or sign in an LSE, an off-by-one in
the iteration count, a dropped adjoint term, a transposed plan, a band index
error) fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import workloads
from tests import dense_surrogate as ds

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ev(s):
    if isinstance(s, (int, float)):
        return float(s)
    return float(eval(s, {"__builtins__": {}}, {"ln": math.log, "sqrt": math.sqrt}))


def _rand(B, H, L, d, seed, **kw):
    x = workloads.draw(B, H, L, d, seed=seed, **kw)
    f = lambda t: None if t is None else t.double().numpy()
    return f(x["q"]), f(x["k"]), f(x["v"]), f(x["dO"]), x["mask"]


def _dense_scores(q, k, eps):
    d = q.shape[-1]
    return (q @ np.swapaxes(k, -1, -2)) / (math.sqrt(d) * eps)


def _band_to_dense(band, W):
    L = band.shape[0]
    out = np.zeros((L, L))
    for i in range(L):
        for t in range(2 * W + 1):
            j = i - W + t
            if 0 <= j < L:
                out[i, j] = band[i, t]
    return out


# --------------------------------------------------------------------------
# worked example and closed forms
# --------------------------------------------------------------------------

def test_golden_2x2_hand_derived(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "sinkhorn_2x2.json")))
    q = np.array([[[[_ev(x) for x in r] for r in g["q"]]]])
    k = np.array([[[[_ev(x) for x in r] for r in g["k"]]]])
    v = np.array([[[[_ev(x) for x in r] for r in g["v"]]]])
    o, st = oracle_mod.forward(q, k, v, W=g["W"], eps=_ev(g["eps"]), T=g["T"], R=g["R"])
    names = ["u0", "v0", "u1", "v1", "u2", "v2"]
    for r, nm in enumerate(names):
        np.testing.assert_allclose(st[0, 0, r], [_ev(x) for x in g[nm]], rtol=0, atol=1e-14,
                                   err_msg=nm)
    np.testing.assert_allclose(o[0, 0], [[_ev(x) for x in r] for r in g["O"]], atol=1e-14)
    band, _, _ = oracle_mod.plan(q, k, st, 2, 2, W=1, eps=_ev(g["eps"]))
    np.testing.assert_allclose(_band_to_dense(band[0, 0], 1),
                               [[_ev(x) for x in r] for r in g["P22"]], atol=1e-14)
    # the base and the tail are the same iteration: T=1, R=1 lands on (u2, v2)
    o1, st1 = oracle_mod.forward(q, k, v, W=1, eps=_ev(g["eps"]), T=1, R=1)
    np.testing.assert_allclose(st1[0, 0, 2], [_ev(x) for x in g["u2"]], atol=1e-14)
    np.testing.assert_allclose(o1, o, atol=1e-14)
    # the limit has a closed form (cross ratio preserved by diagonal scaling)
    _, stl = oracle_mod.forward(q, k, v, W=1, eps=_ev(g["eps"]), T=60, R=2)
    band, _, _ = oracle_mod.plan(q, k, stl, 2, 2, W=1, eps=_ev(g["eps"]))
    assert abs(band[0, 0, 0, 1] - _ev(g["limit_p00"])) < 1e-14


def test_golden_dustbin_one_token_hand_derived(oracle_mod):
    """One real token and the dustbin: the augmented 2 x 2 problem solved in exact
    rationals, including the value cotangents of the token and of the dustbin."""
    g = json.load(open(os.path.join(GOLDEN, "dustbin_1token.json")))
    arr = lambda key: np.array([[[[_ev(x) for x in r] for r in g[key]]]])
    q, k, v, dO = arr("q"), arr("k"), arr("v"), arr("dO")
    vd = np.array([[_ev(x) for x in g["v_dust"]]])
    kw = dict(W=g["W"], eps=_ev(g["eps"]), R=g["R"], dustbin=True, dustbin_score=g["dustbin_score"])
    o, st = oracle_mod.forward(q, k, v, T=g["T"], v_dust=vd, **kw)
    for r, nm in enumerate(["u0", "v0", "u1", "v1", "u2", "v2"]):
        np.testing.assert_allclose(st[0, 0, r], [_ev(x) for x in g[nm]], rtol=0, atol=1e-14,
                                   err_msg=nm)
    np.testing.assert_allclose(o[0, 0], [[_ev(x) for x in r] for r in g["O"]], atol=1e-14)
    for s in ("direct", "one_reference"):
        _, _, dv, dvd = oracle_mod.backward(q, k, v, st, dO, v_dust=vd, schedule=s, **kw)
        np.testing.assert_allclose(dv[0, 0], [[_ev(x) for x in r] for r in g["dV"]], atol=1e-14)
        np.testing.assert_allclose(dvd[0], [_ev(x) for x in g["dv_dust"]], atol=1e-14)


def test_T0_rows_are_softmax(oracle_mod):
    """T = 0: the base is zero, so P^(1,0) is the row softmax of the masked band
    scores (a library routine), u0 = v0 = 0."""
    q, k, v, _, mask = _rand(2, 2, 40, 8, seed=3, mask_kind="holes")
    W, eps = 5, 0.7
    _, st = oracle_mod.forward(q, k, v, W=W, eps=eps, T=0, R=2, mask=mask)
    assert np.all(st[:, :, 0] == 0) and np.all(st[:, :, 1] == 0)
    band, _, _ = oracle_mod.plan(q, k, st, 1, 0, W=W, eps=eps, mask=mask)
    S = torch.tensor(_dense_scores(q, k, eps))
    L = q.shape[2]
    idx = torch.arange(L)
    for b in range(2):
        valid = torch.tensor(mask[b].numpy()).bool()
        sup = ((idx[:, None] - idx[None, :]).abs() <= W) & valid[:, None] & valid[None, :]
        for h in range(2):
            sm = torch.softmax(S[b, h].masked_fill(~sup, float("-inf")), dim=1)
            sm = torch.where(valid[:, None], sm, torch.zeros(()))
            np.testing.assert_allclose(_band_to_dense(band[b, h], W), sm.numpy(), atol=1e-15)


def test_W0_identity_closed_form(oracle_mod):
    """W = 0: the support is the diagonal, every plan is the identity, O = V,
    dV = dO and dQ = dK = 0 exactly; u + v = -S_ii."""
    q, k, v, dO, _ = _rand(1, 2, 33, 16, seed=5)
    o, st = oracle_mod.forward(q, k, v, W=0, eps=0.3, T=4, R=2)
    np.testing.assert_allclose(o, v, atol=1e-13)
    Sii = np.einsum("bhid,bhid->bhi", q, k) / (4.0 * 0.3)
    np.testing.assert_allclose(st[:, :, 4] + st[:, :, 5], -Sii, atol=1e-12)
    for sched in ("direct", "one_reference"):
        dq, dk, dv, _ = oracle_mod.backward(q, k, v, st, dO, W=0, eps=0.3, schedule=sched)
        np.testing.assert_allclose(dv, dO, atol=1e-13)
        assert np.abs(dq).max() < 1e-12 and np.abs(dk).max() < 1e-12


def test_dense_zero_keys_uniform_plan(oracle_mod):
    """K = 0 on a dense support: S = 0, every plan is 1/n, O_i = mean of V."""
    q, _, v, dO, mask = _rand(2, 1, 24, 8, seed=7, valid_len=(10, 24))
    k = np.zeros_like(q)
    o, st = oracle_mod.forward(q, k, v, W=100, eps=1.0, T=3, R=2, mask=mask)
    for b in range(2):
        m = mask[b].numpy().astype(bool)
        mean = v[b, 0, m].mean(axis=0)
        np.testing.assert_allclose(o[b, 0, m], np.broadcast_to(mean, o[b, 0, m].shape),
                                   atol=1e-14)
        assert np.all(o[b, 0, ~m] == 0)
    dq, _, _, _ = oracle_mod.backward(q, k, v, st, dO, W=100, eps=1.0, mask=mask)
    assert np.abs(dq).max() < 1e-14


# --------------------------------------------------------------------------
# invariants of every iterate
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dustbin", [False, True])
def test_marginals_of_every_iterate(oracle_mod, dustbin):
    """u^(r) normalises the rows of P^(r,r-1); v^(r) normalises the columns of
    P^(r,r) (including the dustbin row and column)."""
    q, k, v, _, mask = _rand(1, 2, 70, 8, seed=11, mask_kind="holes")
    W, eps, R = 6, 0.5, 3
    _, st = oracle_mod.forward(q, k, v, W=W, eps=eps, T=2, R=R, mask=mask, dustbin=dustbin,
                               dustbin_score=-1.5)
    m = mask[0].numpy().astype(bool)
    for r in range(1, R + 1):
        for (a, b, axis) in ((r, r - 1, "row"), (r, r, "col")):
            band, dcol, drow = oracle_mod.plan(q, k, st, a, b, W=W, eps=eps, R=R, mask=mask,
                                               dustbin=dustbin, dustbin_score=-1.5)
            for h in range(2):
                P = _band_to_dense(band[0, h], W)
                if dustbin:
                    P = np.block([[P, dcol[0, h][:, None]], [drow[0, h][None, :]]])
                mm = np.concatenate([m, [True]]) if dustbin else m
                s = P.sum(axis=1 if axis == "row" else 0)
                np.testing.assert_allclose(s[mm], 1.0, atol=1e-13)
                assert np.all(s[~mm] == 0)


def test_base_and_tail_are_one_iteration(oracle_mod):
    """Running T+1 base iterations shifts the tail by one step: the duals after
    step r of (T+1) equal those after step r+1 of T.  With the T = 0 softmax pin
    this fixes the iteration count by induction."""
    q, k, v, _, mask = _rand(1, 1, 50, 8, seed=13, valid_len=(30, 50))
    kw = dict(W=4, eps=0.6, R=3, mask=mask)
    _, a = oracle_mod.forward(q, k, v, T=5, **kw)
    _, b = oracle_mod.forward(q, k, v, T=6, **kw)
    np.testing.assert_array_equal(b[:, :, 0:6], a[:, :, 2:8])


def test_converges_to_doubly_stochastic(oracle_mod):
    """Large T: P^(R,R) is doubly stochastic, and log P - S is additive
    (u_i + v_j), which characterises the Sinkhorn scaling uniquely."""
    q, k, v, _, _ = _rand(1, 1, 60, 8, seed=17)
    W, eps = 7, 1.0
    _, st = oracle_mod.forward(q, k, v, W=W, eps=eps, T=400, R=2)
    band, _, _ = oracle_mod.plan(q, k, st, 2, 2, W=W, eps=eps)
    P = _band_to_dense(band[0, 0], W)
    np.testing.assert_allclose(P.sum(1), 1.0, atol=1e-10)
    np.testing.assert_allclose(P.sum(0), 1.0, atol=1e-13)


def test_gauge_invariance(oracle_mod):
    """A constant added to the frozen v0 is absorbed by u^(1): every plan, O and
    gradient is unchanged.  A per-row constant added to S (extra coordinate,
    scale kept) is absorbed by the u-updates in the same way."""
    q, k, v, dO, mask = _rand(1, 2, 40, 8, seed=19, mask_kind="holes")
    W, eps = 5, 0.8
    o, st = oracle_mod.forward(q, k, v, W=W, eps=eps, T=3, mask=mask)
    base = st[:, :, 0:2].copy()
    base[:, :, 1] += np.where(mask.numpy()[:, None, :] > 0, 0.37, 0.0)
    o2, st2 = oracle_mod.forward(q, k, v, W=W, eps=eps, T=3, mask=mask, base=base)
    np.testing.assert_allclose(o2, o, atol=1e-13)
    g1 = oracle_mod.backward(q, k, v, st, dO, W=W, eps=eps, mask=mask)
    g2 = oracle_mod.backward(q, k, v, st2, dO, W=W, eps=eps, mask=mask)
    for x, y in zip(g1[:3], g2[:3]):
        np.testing.assert_allclose(x, y, atol=1e-12)
    # per-row constants: append kappa_i/c to q and a 1 to k, keep c fixed
    d = q.shape[-1]
    c = 1.0 / (math.sqrt(d) * eps)
    eps2 = 1.0 / (math.sqrt(d + 1) * c)
    kappa = np.random.default_rng(0).normal(size=q.shape[:-1]) * 3.0
    q2 = np.concatenate([q, (kappa / c)[..., None]], -1)
    k2 = np.concatenate([k, np.ones(k.shape[:-1] + (1,))], -1)
    v2 = np.concatenate([v, np.zeros(v.shape[:-1] + (1,))], -1)
    o3, _ = oracle_mod.forward(q2, k2, v2, W=W, eps=eps2, T=3, mask=mask)
    np.testing.assert_allclose(o3[..., :d], o, atol=1e-12)


def test_tail_padding_equals_truncation(oracle_mod):
    """A tail-padded problem equals the truncated problem, bit for bit, and its
    padded rows/columns are exactly zero."""
    q, k, v, dO, _ = _rand(1, 1, 64, 8, seed=23)
    n = 45
    mask = np.zeros((1, 64), np.uint8)
    mask[0, :n] = 1
    kw = dict(W=6, eps=0.7, T=4)
    o, st = oracle_mod.forward(q, k, v, mask=mask, **kw)
    ot, stt = oracle_mod.forward(q[:, :, :n], k[:, :, :n], v[:, :, :n], **kw)
    np.testing.assert_array_equal(o[:, :, :n], ot)
    np.testing.assert_array_equal(st[..., :n], stt)
    assert np.all(o[:, :, n:] == 0) and np.all(st[..., n:] == 0)
    g = oracle_mod.backward(q, k, v, st, dO, mask=mask, **{k_: kw[k_] for k_ in ("W", "eps")})
    gt = oracle_mod.backward(q[:, :, :n], k[:, :, :n], v[:, :, :n], stt, dO[:, :, :n],
                             **{k_: kw[k_] for k_ in ("W", "eps")})
    for x, y in zip(g[:3], gt[:3]):
        np.testing.assert_array_equal(x[:, :, :n], y)
        assert np.all(x[:, :, n:] == 0)


# --------------------------------------------------------------------------
# the backward: autograd, finite differences, schedules, orbit identity
# --------------------------------------------------------------------------

CASES = [
    # (L, d, W, eps, T, R, mask_kind, dustbin)
    (17, 4, 3, 0.7, 3, 2, None, False),
    (32, 8, 5, 0.5, 6, 2, "holes", False),
    (24, 8, 30, 1.0, 2, 2, None, False),      # W >= L: dense
    (20, 4, 4, 0.9, 0, 2, None, False),       # T = 0
    (19, 4, 3, 0.8, 3, 1, "holes", False),    # R = 1
    (21, 4, 3, 0.8, 2, 4, None, False),       # R = 4
    (18, 4, 3, 0.7, 3, 2, None, True),        # dustbin
    (26, 8, 4, 0.6, 4, 2, "holes", True),     # dustbin + holes
    (22, 4, 3, 0.8, 2, 6, "holes", False),    # R = 6: more terms than one dS sweep takes
    (20, 4, 4, 0.9, 1, 9, None, True),        # R = 9 with the dustbin
    (16, 4, 2, 1.0, 0, 9, "holes", False),    # T = 0, R = 9: full backpropagation
]


@pytest.mark.parametrize("case", CASES)
def test_matches_dense_autograd(oracle_mod, case):
    """Forward, duals and both backward schedules equal exact autodiff of the
    same surrogate (dense float64 torch), as in the pages' exactness check."""
    L, d, W, eps, T, R, mk, db = case
    q, k, v, dO, mask = _rand(1, 2, L, d, seed=L * 7 + W, mask_kind=mk)
    rng = np.random.default_rng(L)
    vd = rng.normal(size=(2, d)) if db else None
    kw = dict(W=W, eps=eps, T=T, R=R, dustbin=db, dustbin_score=-1.3)
    o, st = oracle_mod.forward(q, k, v, mask=mask, v_dust=vd, **kw)
    grads = {s: oracle_mod.backward(q, k, v, st, dO, mask=mask, v_dust=vd, schedule=s,
                                    **{x: kw[x] for x in ("W", "eps", "R", "dustbin",
                                                          "dustbin_score")})
             for s in ("direct", "one_reference")}
    for h in range(2):
        m = None if mask is None else mask[0].numpy()
        ro, rst, rdq, rdk, rdv, rdvd = ds.surrogate_and_grads(
            q[0, h], k[0, h], v[0, h], dO[0, h], mask=m, v_dust=None if vd is None else vd[h],
            **kw)
        np.testing.assert_allclose(o[0, h], ro, atol=1e-12)
        np.testing.assert_allclose(st[0, h], rst, atol=1e-11)
        for s, (dq, dk, dv, dvd) in grads.items():
            scale = max(np.abs(rdq).max(), np.abs(rdk).max(), 1.0)
            np.testing.assert_allclose(dq[0, h], rdq, atol=1e-10 * scale, err_msg=s)
            np.testing.assert_allclose(dk[0, h], rdk, atol=1e-10 * scale, err_msg=s)
            np.testing.assert_allclose(dv[0, h], rdv, atol=1e-11, err_msg=s)
            if db:
                np.testing.assert_allclose(dvd[h], rdvd, atol=1e-11, err_msg=s)


@pytest.mark.parametrize("d,dustbin", [(4, False), (64, False), (8, True)])
def test_frozen_base_finite_differences(oracle_mod, d, dustbin):
    """Central differences of F = <dO, O> along random directions, with the
    stopped base held at its unperturbed value (the surrogate's derivative)."""
    L, W, eps, T = 20, 3, 0.8, 5
    q, k, v, dO, mask = _rand(1, 1, L, d, seed=29 + d, mask_kind="holes")
    kw = dict(W=W, eps=eps, T=T, mask=mask, dustbin=dustbin, dustbin_score=-0.7)
    o, st = oracle_mod.forward(q, k, v, **kw)
    base = st[:, :, 0:2].copy()
    dq, dk, dv, _ = oracle_mod.backward(q, k, v, st, dO, W=W, eps=eps, mask=mask,
                                        dustbin=dustbin, dustbin_score=-0.7)
    rng = np.random.default_rng(d)
    h = 1e-5

    def F(qq, kk, vv):
        oo, _ = oracle_mod.forward(qq, kk, vv, base=base, **kw)
        return float((oo * dO).sum())

    for _ in range(3):
        eq, ek, ev = (rng.normal(size=q.shape) for _ in range(3))
        fd = (F(q + h * eq, k + h * ek, v + h * ev) - F(q - h * eq, k - h * ek, v - h * ev)) / (2 * h)
        an = float((dq * eq).sum() + (dk * ek).sum() + (dv * ev).sum())
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)


# --------------------------------------------------------------------------
# the dustbin score's cotangent (one learned dustbin token, gist.science/de
# section 2.3): the sum of dS over the dustbin column, row and corner
# --------------------------------------------------------------------------

DSCORE_CASES = [
    # (L, d, W, eps, T, R, mask_kind)
    (18, 4, 3, 0.7, 3, 2, None),
    (26, 8, 4, 0.6, 4, 2, "holes"),
    (15, 4, 20, 1.0, 2, 1, None),     # W >= L: dense
    (21, 4, 3, 0.8, 2, 3, "holes"),
    (16, 4, 2, 0.9, 0, 2, None),      # T = 0
]


@pytest.mark.parametrize("case", DSCORE_CASES)
def test_dustbin_score_cotangent_matches_autograd(oracle_mod, case):
    L, d, W, eps, T, R, mk = case
    q, k, v, dO, mask = _rand(1, 2, L, d, seed=3 * L + W, mask_kind=mk)
    vd = np.random.default_rng(L + 1).normal(size=(2, d))
    sc = -0.9
    kw = dict(W=W, eps=eps, R=R, dustbin=True, dustbin_score=sc)
    o, st = oracle_mod.forward(q, k, v, T=T, mask=mask, v_dust=vd, **kw)
    m = None if mask is None else mask[0].numpy()
    ref = sum(ds.dustbin_score_grad(q[0, h], k[0, h], v[0, h], dO[0, h], v_dust=vd[h], W=W,
                                    eps=eps, T=T, R=R, mask=m, dustbin_score=sc)
              for h in range(2))
    assert abs(ref) > 1e-3  # the pin has something to check
    for s in ("direct", "one_reference"):
        g = oracle_mod.backward(q, k, v, st, dO, mask=mask, v_dust=vd, schedule=s,
                                score_grad=True, **kw)[4]
        assert abs(g - ref) <= 1e-10 * max(1.0, abs(ref)), (s, g, ref)


def test_dustbin_score_cotangent_finite_differences(oracle_mod):
    """Central difference of F = <dO, O> in the dustbin score, the stopped base
    held at its unperturbed value."""
    L, d, W, eps, T, R = 22, 8, 3, 0.8, 4, 2
    q, k, v, dO, mask = _rand(2, 2, L, d, seed=77, mask_kind="holes")
    vd = np.random.default_rng(5).normal(size=(2, d))
    sc, h = -1.1, 1e-5
    kw = dict(W=W, eps=eps, R=R, mask=mask, dustbin=True, v_dust=vd)
    o, st = oracle_mod.forward(q, k, v, T=T, dustbin_score=sc, **kw)
    base = st[:, :, 0:2].copy()
    g = oracle_mod.backward(q, k, v, st, dO, dustbin_score=sc, score_grad=True, **kw)[4]

    def F(s):
        oo, _ = oracle_mod.forward(q, k, v, T=T, base=base, dustbin_score=s, **kw)
        return float((oo * dO).sum())

    fd = (F(sc + h) - F(sc - h)) / (2 * h)
    assert abs(fd - g) <= 1e-7 * max(1.0, abs(g)), (fd, g)


def test_dustbin_score_cotangent_is_zero_without_a_dustbin(oracle_mod):
    q, k, v, dO, mask = _rand(1, 1, 12, 4, seed=2)
    o, st = oracle_mod.forward(q, k, v, W=2, eps=1.0, T=2, R=2)
    assert oracle_mod.backward(q, k, v, st, dO, W=2, eps=1.0, R=2, score_grad=True)[4] == 0.0


def test_one_reference_equals_direct(oracle_mod):
    q, k, v, dO, mask = _rand(2, 2, 90, 16, seed=31, valid_len=(60, 90))
    kw = dict(W=9, eps=0.5, R=2, mask=mask)
    _, st = oracle_mod.forward(q, k, v, T=7, **kw)
    a = oracle_mod.backward(q, k, v, st, dO, schedule="direct", **kw)
    b = oracle_mod.backward(q, k, v, st, dO, schedule="one_reference", **kw)
    for x, y in zip(a[:3], b[:3]):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-12 * max(1.0, np.abs(x).max()))


def test_orbit_identity(oracle_mod):
    """Every staircase plan equals P^(2,2) rescaled by exp(u^(a) - u^(2)) on rows
    and exp(v^(b) - v^(2)) on columns (technical summary section 2.2)."""
    q, k, v, _, mask = _rand(1, 1, 64, 8, seed=37, mask_kind="holes")
    kw = dict(W=6, eps=0.6, R=2, mask=mask)
    _, st = oracle_mod.forward(q, k, v, T=4, **kw)
    ref, _, _ = oracle_mod.plan(q, k, st, 2, 2, **kw)
    W = 6
    for a, b in ((2, 1), (1, 1), (1, 0)):
        P, _, _ = oracle_mod.plan(q, k, st, a, b, **kw)
        du = np.exp(st[0, 0, 2 * a] - st[0, 0, 4])
        dv = np.exp(st[0, 0, 2 * b + 1] - st[0, 0, 5])
        L = 64
        for i in range(L):
            for t in range(2 * W + 1):
                j = i - W + t
                if 0 <= j < L and ref[0, 0, i, t] != 0:
                    x = ref[0, 0, i, t] * du[i] * dv[j]
                    assert abs(P[0, 0, i, t] - x) <= 1e-13 * abs(x)
                else:
                    assert P[0, 0, i, t] == 0


# --------------------------------------------------------------------------
# work count: O(L W)
# --------------------------------------------------------------------------

@pytest.mark.parametrize("L,W,T,db", [(100, 7, 3, False), (257, 20, 5, False), (64, 70, 2, False),
                                      (90, 5, 4, True)])
def test_work_is_linear_in_support(oracle_mod, L, W, T, db):
    """The forward visits each support entry once per half-sweep plus once for
    the output: (2T + 2R) |Omega_aug| + |Omega rows of real tokens|; the
    backward visits a fixed multiple of |Omega_aug| that depends on neither L,
    W nor T."""
    R = 2
    q, k, v, dO, _ = _rand(1, 1, L, 4, seed=L)
    n = L
    band = n * (2 * W + 1) - W * (W + 1) if n > W else n * n
    aug = band + (2 * n + 1 if db else 0)
    real_rows = band + (n if db else 0)
    _, st, vis = oracle_mod.forward(q, k, v, W=W, eps=1.0, T=T, R=R, dustbin=db, count=True)
    assert oracle_mod.support_size(L, W, dustbin=db) == aug
    assert vis[0, 0] == (2 * T + 2 * R) * aug + real_rows
    _, bvis = oracle_mod.backward(q, k, v, st, dO, W=W, eps=1.0, R=R, dustbin=db,
                                  schedule="one_reference", count=True)
    assert bvis[0, 0] == 5 * aug
    _, bvis = oracle_mod.backward(q, k, v, st, dO, W=W, eps=1.0, R=R, dustbin=db,
                                  schedule="direct", count=True)
    assert bvis[0, 0] == 8 * aug


# --------------------------------------------------------------------------
# random small configurations (property-based): every parameter at once
# --------------------------------------------------------------------------

from hypothesis import HealthCheck, given, settings, strategies as st_


@settings(max_examples=60, deadline=None, derandomize=True,
          suppress_health_check=[HealthCheck.too_slow])
@given(L=st_.integers(1, 20), d=st_.sampled_from([1, 2, 3, 4, 8]), W=st_.integers(0, 22),
       eps=st_.floats(0.4, 1.5), T=st_.integers(0, 4), R=st_.integers(1, 5),
       dustbin=st_.booleans(), seed=st_.integers(0, 2 ** 31 - 1))
def test_random_configurations_match_dense_autograd(oracle_mod, L, d, W, eps, T, R, dustbin, seed):
    """Any band (W = 0 up to dense), length (down to one token), head size,
    depth, random mask (down to a single valid token, or none) and dustbin: the
    forward, the duals and both backward schedules equal exact autodiff of the
    dense surrogate, and masked tokens carry exact zeros."""
    rng = np.random.default_rng(seed)
    q, k, v, dO = (rng.normal(size=(1, 1, L, d)) for _ in range(4))
    mask = (rng.random((1, L)) < rng.uniform(0.3, 1.0)).astype(np.uint8)
    vd = rng.normal(size=(1, d)) if dustbin else None
    kw = dict(W=W, eps=eps, R=R, dustbin=dustbin, dustbin_score=float(rng.uniform(-3, 1)))
    o, st = oracle_mod.forward(q, k, v, T=T, mask=mask, v_dust=vd, **kw)
    grads = {s: oracle_mod.backward(q, k, v, st, dO, mask=mask, v_dust=vd, schedule=s, **kw)
             for s in ("direct", "one_reference")}
    m = mask[0].astype(bool)
    if not m.any():  # nothing valid: every output and dual is zero
        assert not o.any() and not st[..., :L].any()
        for dq, dk, dv, _ in grads.values():
            assert not dq.any() and not dk.any() and not dv.any()
        return
    ro, rst, rdq, rdk, rdv, rdvd = ds.surrogate_and_grads(
        q[0, 0], k[0, 0], v[0, 0], dO[0, 0], mask=mask[0], T=T,
        v_dust=None if vd is None else vd[0], **kw)
    np.testing.assert_allclose(o[0, 0], ro, atol=1e-11)
    np.testing.assert_allclose(st[0, 0], rst, atol=1e-10)
    for s, (dq, dk, dv, dvd) in grads.items():
        scale = max(np.abs(rdq).max(), np.abs(rdk).max(), 1.0)
        np.testing.assert_allclose(dq[0, 0], rdq, atol=1e-9 * scale, err_msg=s)
        np.testing.assert_allclose(dk[0, 0], rdk, atol=1e-9 * scale, err_msg=s)
        np.testing.assert_allclose(dv[0, 0], rdv, atol=1e-10, err_msg=s)
        assert not dq[0, 0, ~m].any() and not dk[0, 0, ~m].any() and not dv[0, 0, ~m].any()
        if dustbin:
            np.testing.assert_allclose(dvd[0], rdvd, atol=1e-10, err_msg=s)
