"""Pins of the full-backpropagation gradients, the tail-depth-0 gradients and
the bias certificate (Block-Wise Differentiable Sinkhorn Attention,
gist.science/de technical summary: section 3, a posteriori bias certificate and
tail-depth selection at a tolerance; section 4.1, bias decay of tail gradients
against full backpropagation through time).

Every oracle quantity is checked against the independent dense float64 autograd
implementation in ``tests/dense_surrogate.py``."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads
from tests import dense_surrogate as ds


def _case(L=40, d=8, seed=3, holes=True):
    x = workloads.draw(1, 1, L, d, dtype="f32", seed=seed, mask_kind="holes" if holes else None)
    q, k, v, dO = (x[n].double().numpy() for n in ("q", "k", "v", "dO"))
    m = None if x["mask"] is None else x["mask"].numpy()
    return q, k, v, dO, m


def _dense(q, k, v, dO, m, **kw):
    mask = None if m is None else m[0]
    _, _, dq, dk, dv, _ = ds.surrogate_and_grads(q[0, 0], k[0, 0], v[0, 0], dO[0, 0], mask=mask, **kw)
    return dq, dk, dv


@pytest.mark.parametrize("T,R,W", [(3, 2, 5), (0, 3, 4), (4, 1, 39)])
def test_full_bptt_matches_dense_autograd_through_the_base(T, R, W):
    q, k, v, dO, m = _case()
    _, _, g = oracle.full_bptt(q, k, v, dO, N=T + R, W=W, eps=0.7, mask=m)
    ref = _dense(q, k, v, dO, m, W=W, eps=0.7, T=T, R=R, stop_base=False)
    for a, b in zip(g, ref):
        np.testing.assert_allclose(a[0, 0], b, rtol=0, atol=1e-10 * max(1.0, np.abs(b).max()))


def test_full_bptt_is_the_zero_base_surrogate_in_the_dense_implementation():
    # the identity behind full_bptt, checked where the oracle plays no part
    q, k, v, dO, m = _case(seed=7)
    a = _dense(q, k, v, dO, m, W=6, eps=1.0, T=3, R=2, stop_base=False)
    b = _dense(q, k, v, dO, m, W=6, eps=1.0, T=0, R=5, stop_base=True)
    for x, y in zip(a, b):
        np.testing.assert_allclose(x, y, rtol=0, atol=1e-12 * max(1.0, np.abs(y).max()))


@pytest.mark.parametrize("W", [0, 3, 39])
def test_stopped_gradients_match_dense_tail_depth_zero(W):
    q, k, v, dO, m = _case(seed=11)
    g = oracle.stopped_gradients(q, k, v, dO, N=5, W=W, eps=0.9, mask=m)
    ref = _dense(q, k, v, dO, m, W=W, eps=0.9, T=5, R=0)
    for a, b in zip(g, ref):
        np.testing.assert_allclose(a[0, 0], b, rtol=0, atol=1e-10 * max(1.0, np.abs(b).max()))


def test_certificate_matches_dense_remainders_and_selects_depth():
    q, k, v, dO, m = _case(L=48, seed=5)
    N, W, eps = 8, 6, 1.0
    Rs = (0, 1, 2, 4, N)
    eta, rstar = oracle.bias_certificate(q, k, v, dO, N=N, Rs=Rs, tau=1e-5, W=W, eps=eps, mask=m)
    full = _dense(q, k, v, dO, m, W=W, eps=eps, T=0, R=N)
    ref = np.sqrt(sum(np.sum(x * x) for x in full))
    for R in Rs:
        g = _dense(q, k, v, dO, m, W=W, eps=eps, T=N - R, R=R)
        e = np.sqrt(sum(np.sum((a - b) ** 2) for a, b in zip(g, full))) / ref
        assert eta[R] == pytest.approx(e, rel=1e-8, abs=1e-13)
    assert eta[N] == 0.0                      # R = N is full backpropagation itself
    assert eta[0] > eta[1] > eta[2]           # the bias decays with the tail depth
    assert rstar == min(R for R in Rs if eta[R] <= 1e-5)
    # a tolerance between two certificates selects the deeper of the two
    tau = 0.5 * (eta[1] + eta[2])
    _, r2 = oracle.bias_certificate(q, k, v, dO, N=N, Rs=Rs, tau=tau, W=W, eps=eps, mask=m)
    assert r2 == 2
