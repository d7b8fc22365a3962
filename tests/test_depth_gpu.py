"""Tail depth on the GPU: depth 0 (every iteration stopped), full
backpropagation (T = 0, R = N) and the a-posteriori bias certificate
(gist.science/de section 3, section 4.1), each against the oracle on the same
seeded inputs.

Depth 0 runs N iterations and holds every dual constant, so its forward equals
the oracle's forward with N - 1 stopped iterations and one tail step (the duals
after N iterations sit in tail row 1 there), and its gradients are the
oracle's ``stopped_gradients``.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import parity

pytestmark = pytest.mark.gpu


DEPTH0 = [
    # (L, W, eps, N, dtype, mask_kind / valid_len)
    (200, 17, 0.6, 6, "f32", "holes"),
    (130, 200, 1.0, 1, "f32", None),
    (520, 64, 0.8, 5, "bf16", (300, 520)),
    (300, 256, 1.0, 3, "bf16", "holes"),
]


@pytest.mark.parametrize("case", DEPTH0, ids=lambda c: "L{}_W{}_N{}_{}".format(c[0], c[1], c[3], c[4]))
def test_tail_depth_zero(case):
    import banded_log_domain_b200 as sa

    L, W, eps, N, dtype, mk = case
    B, H = 2, 2
    x = parity.draw_case(B, H, L, dtype=dtype, seed=7 * L + W,
                         mask_kind=mk if isinstance(mk, str) else None,
                         valid_len=mk if isinstance(mk, tuple) else None)
    d = parity.to_dev(x)
    o, st = sa.sinkhorn_attn_fwd(d["q"], d["k"], d["v"], W=W, eps=eps, T=N, R=0, mask=d["mask"])
    assert tuple(st.shape) == (B, H, 2, L)
    grads = {s: sa.sinkhorn_attn_bwd(d["q"], d["k"], d["v"], o, d["dO"], st, W=W, eps=eps, R=0,
                                     mask=d["mask"], schedule=s)
             for s in ("one_reference", "direct")}
    torch.cuda.synchronize()
    np_ = lambda t: t.detach().float().cpu().double().numpy()

    ro, rst = oracle.forward(x["q"], x["k"], x["v"], W=W, eps=eps, T=N - 1, R=1, mask=x["mask"])
    rg = oracle.stopped_gradients(x["q"], x["k"], x["v"], x["dO"], N=N, W=W, eps=eps,
                                  mask=x["mask"])
    vm = parity.valid_mask(x, B, L)
    m = np.broadcast_to(vm[:, None, None, :], (B, H, 2, L))
    err = np.abs(np_(st) - rst[:, :, 2:4])[m].max()
    assert err <= parity.DUAL_ATOL[dtype], f"duals {err}"
    mo = np.broadcast_to(vm[:, None, :, None], (B, H, L, 64))
    tol = parity.REL_L2[dtype]
    e = parity.rel_l2(np_(o)[mo], ro[mo])
    assert e <= tol, f"O {e}"
    assert np.all(np_(o)[~mo] == 0)
    for s, g in grads.items():
        for name, gt, rt in zip(("dQ", "dK", "dV"), g[:3], rg):
            e = parity.rel_l2(np_(gt)[mo], rt[mo])
            assert e <= tol, f"{s} {name} rel-l2 {e}"
            assert np.all(np_(gt)[~mo] == 0), f"{s} masked {name} not zero"


def test_tail_depth_zero_dustbin_gradients():
    # every dual constant: dv_dust = sum_i P_(i,dustbin) dO_i and the score's
    # cotangent sum_i P_(i,dustbin) <dO_i, v_dust> (G is zero on the dustbin row)
    import banded_log_domain_b200 as sa

    L, W, eps, N, B, H = 150, 9, 0.8, 4, 2, 2
    x = parity.draw_case(B, H, L, dtype="f32", seed=19, mask_kind="holes", dustbin=True,
                         v_dust_random=True)
    d = parity.to_dev(x)
    kw = dict(W=W, eps=eps, dustbin=True, dustbin_score=-1.4)
    o, st = sa.sinkhorn_attn_fwd(d["q"], d["k"], d["v"], T=N, R=0, mask=d["mask"],
                                 v_dust=d["v_dust"], **kw)
    dsc = torch.zeros(1, dtype=torch.float32, device="cuda")
    _, _, _, dvd = sa.sinkhorn_attn_bwd(d["q"], d["k"], d["v"], o, d["dO"], st, R=0,
                                        mask=d["mask"], v_dust=d["v_dust"], d_dust_score=dsc, **kw)
    torch.cuda.synchronize()
    _, rst = oracle.forward(x["q"], x["k"], x["v"], T=N - 1, R=1, mask=x["mask"],
                            v_dust=x["v_dust"], **kw)
    _, dcol, _ = oracle.plan(x["q"], x["k"], rst, 1, 1, R=1, mask=x["mask"], **kw)
    dO = x["dO"].double().numpy()
    vd = x["v_dust"].double().numpy()
    r_dvd = np.einsum("bhl,bhld->hd", dcol, dO)
    r_dsc = float(np.einsum("bhl,bhld,hd->", dcol, dO, vd))
    assert parity.rel_l2(dvd.double().cpu().numpy(), r_dvd) <= 1e-4
    assert abs(float(dsc[0]) - r_dsc) <= 1e-4 * max(abs(r_dsc), 1e-3)


def test_full_backpropagation_matches_oracle():
    # T = 0, R = N = 12: 24 modifier terms, three blocks of the dS sweep
    L, W, eps, N = 260, 30, 0.7, 12
    for dtype in ("f32", "bf16"):
        x = parity.draw_case(2, 2, L, dtype=dtype, seed=5, valid_len=(160, 260))
        kw = dict(W=W, eps=eps, T=0, R=N)
        g = parity.gpu_run(x, schedules=("one_reference", "direct"), **kw)
        r = parity.oracle_run(x, **kw)  # T = 0, R = N: oracle.full_bptt's solve
        parity.compare(x, g, r, dtype=dtype, dustbin=False, schedules=("one_reference", "direct"),
                       label=f"full bptt {dtype}")


def test_sq_dist_against_numpy():
    import banded_log_domain_b200 as sa

    gen = torch.Generator().manual_seed(3)
    for dt, n in ((torch.float32, 1_000_003), (torch.bfloat16, 777), (torch.float32, 0)):
        a = torch.randn(n, generator=gen).to(dt)
        b = torch.randn(n, generator=gen).to(dt)
        d2, n2 = sa.sinkhorn_attn_sq_dist(a.cuda(), b.cuda())
        a64, b64 = a.double().numpy(), b.double().numpy()
        assert d2 == pytest.approx(float(np.sum((a64 - b64) ** 2)), rel=1e-12, abs=0)
        assert n2 == pytest.approx(float(np.sum(b64 ** 2)), rel=1e-12, abs=0)


def test_bias_certificate_matches_oracle():
    import banded_log_domain_b200 as sa

    L, W, eps, N, Rs = 300, 20, 1.0, 8, (0, 1, 2, 4)
    x = parity.draw_case(1, 2, L, dtype="f32", seed=11, mask_kind="holes")
    r_eta, _ = oracle.bias_certificate(x["q"], x["k"], x["v"], x["dO"], N=N, Rs=Rs, W=W, eps=eps,
                                       mask=x["mask"])
    assert r_eta[0] > r_eta[1] > r_eta[2] > r_eta[4] > 0
    tau = float(np.sqrt(r_eta[1] * r_eta[2]))  # between eta_1 and eta_2: selects R = 2
    d = parity.to_dev(x)
    for s in ("one_reference", "direct"):
        g_eta, g_sel = sa.bias_certificate(d["q"], d["k"], d["v"], d["dO"], N=N, Rs=Rs, tau=tau,
                                           W=W, eps=eps, mask=d["mask"], schedule=s)
        for R in Rs:
            assert abs(g_eta[R] - r_eta[R]) <= 1e-6 + 1e-3 * r_eta[R], (s, R, g_eta[R], r_eta[R])
        assert g_sel == 2
    # bf16 storage: gradients are rounded to bf16 (unit roundoff 2^-8), which
    # sets a floor of a few 1e-3 under every eta
    xb = parity.draw_case(1, 2, L, dtype="bf16", seed=11, mask_kind="holes")
    rb, _ = oracle.bias_certificate(xb["q"], xb["k"], xb["v"], xb["dO"], N=N, Rs=Rs, W=W, eps=eps,
                                    mask=xb["mask"])
    db = parity.to_dev(xb)
    gb, _ = sa.bias_certificate(db["q"], db["k"], db["v"], db["dO"], N=N, Rs=Rs, W=W, eps=eps,
                                mask=db["mask"])
    for R in Rs:
        assert abs(gb[R] - rb[R]) <= 1e-2, (R, gb[R], rb[R])
