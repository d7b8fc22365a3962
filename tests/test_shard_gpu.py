"""Sequence sharding on one GPU: the ranks of a sequence-sharded problem are
emulated as host threads, each with its own CUDA stream, and their halo
exchanges meet at a host barrier after every sweep (the host orders them: no
kernel waits on another rank's kernel).  The own tokens' results must equal
the unsharded problem's, checked against the oracle with the parity
tolerances and against the unsharded GPU run.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from tests import parity

pytestmark = pytest.mark.gpu


class ThreadExchange:
    """Exchange among ``world`` emulated ranks of one process.  Call k of every
    rank waits until every rank's vector k is final, copies its halos from the
    neighbours' own entries, and waits again so that no rank overwrites a
    vector that another is still reading."""

    def __init__(self, bounds):
        self.bounds = bounds  # per rank (own_lo, own_hi, lo, hi) in global tokens
        self.world = len(bounds)
        self.bar = threading.Barrier(self.world, timeout=120)
        self.views = [None] * self.world
        self.calls = [0] * self.world

    def for_rank(self, r):
        own_lo, own_hi, lo, hi = self.bounds[r]

        def ex(view):
            torch.cuda.current_stream().synchronize()  # this rank's sweep is done
            self.views[r] = view
            self.calls[r] += 1
            self.bar.wait()
            if lo < own_lo:  # tokens [lo, own_lo) are the left neighbour's
                llo = self.bounds[r - 1][2]
                view[:, 0:own_lo - lo].copy_(self.views[r - 1][:, lo - llo:own_lo - llo])
            if own_hi < hi:  # tokens [own_hi, hi) are the right neighbour's
                rlo = self.bounds[r + 1][2]
                view[:, own_hi - lo:hi - lo].copy_(self.views[r + 1][:, own_hi - rlo:hi - rlo])
            torch.cuda.current_stream().synchronize()
            self.bar.wait()

        return ex


def run_sharded(x, world, *, W, eps, T, R, schedule):
    import banded_log_domain_b200 as sa

    d = parity.to_dev(x)
    B, H, Lt, _ = x["q"].shape
    bounds = [sa.shard_bounds(Lt, W, r, world) for r in range(world)]
    ex = ThreadExchange(bounds)
    out = [None] * world
    errors = []

    def rank(r):
        try:
            own_lo, own_hi, lo, hi = bounds[r]
            loc = {k: (None if v is None else
                       (v[:, lo:hi].contiguous() if k == "mask" else v[:, :, lo:hi].contiguous()))
                   for k, v in d.items() if k in ("q", "k", "v", "dO", "mask")}
            kw = dict(W=W, eps=eps, R=R, mask=loc["mask"], halo_lo=own_lo - lo,
                      halo_hi=hi - own_hi, exchange=ex.for_rank(r))
            with torch.cuda.stream(torch.cuda.Stream()):
                o, st = sa.sinkhorn_attn_fwd_sharded(loc["q"], loc["k"], loc["v"], T=T, **kw)
                g = sa.sinkhorn_attn_bwd_sharded(loc["q"], loc["k"], loc["v"], o, loc["dO"], st,
                                                 schedule=schedule, **kw)
                torch.cuda.current_stream().synchronize()
            own = slice(own_lo - lo, own_hi - lo)
            out[r] = (o[:, :, own], st[..., own]) + tuple(t[:, :, own] for t in g)
        except BaseException as e:  # noqa: BLE001 - reported below
            errors.append(e)
            ex.bar.abort()

    ts = [threading.Thread(target=rank, args=(r,)) for r in range(world)]
    for t in ts:
        t.start()
    for t in ts:
        t.join(300)
    assert not errors, errors
    assert len(set(ex.calls)) == 1  # every rank made the same exchanges
    cat = lambda i, dim: torch.cat([o[i] for o in out], dim=dim)
    np_ = lambda t: t.detach().float().cpu().double().numpy()
    res = {"o": np_(cat(0, 2)), "state": np_(cat(1, 3))}
    res[schedule] = (np_(cat(2, 2)), np_(cat(3, 2)), np_(cat(4, 2)), None, None)
    return res, ex.calls[0]


CASES = [
    # (L, W, eps, T, R, dtype, world, mask_kind / valid_len)
    (700, 60, 0.8, 3, 2, "f32", 3, "holes"),
    (520, 33, 1.0, 0, 1, "f32", 2, None),
    (900, 100, 1.0, 4, 2, "bf16", 3, (800, 900)),
    (1024, 256, 1.0, 2, 3, "bf16", 4, None),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "L{}_W{}_R{}_{}_x{}".format(
    c[0], c[1], c[4], c[5], c[6]))
@pytest.mark.parametrize("schedule", ["one_reference", "direct"])
def test_sharded_equals_unsharded(case, schedule):
    L, W, eps, T, R, dtype, world, mk = case
    x = parity.draw_case(1, 2, L, dtype=dtype, seed=L + W,
                         mask_kind=mk if isinstance(mk, str) else None,
                         valid_len=mk if isinstance(mk, tuple) else None)
    kw = dict(W=W, eps=eps, T=T, R=R)
    g, ncalls = run_sharded(x, world, schedule=schedule, **kw)
    assert ncalls == 2 * (T + R) + 2 * R  # one per sweep that produces a dual or cotangent
    r = parity.oracle_run(x, **kw)
    parity.compare(x, g, r, dtype=dtype, dustbin=False, schedules=(schedule,),
                   label=f"sharded x{world} {case}")
    u = parity.gpu_run(x, schedules=(schedule,), **kw)
    tol = parity.REL_L2[dtype]
    for i, name in enumerate(("dQ", "dK", "dV")):
        assert parity.rel_l2(g[schedule][i], u[schedule][i]) <= tol, name
    assert parity.rel_l2(g["o"], u["o"]) <= tol


def test_failing_exchange_is_reported():
    import banded_log_domain_b200 as sa

    x = parity.to_dev(parity.draw_case(1, 1, 64, dtype="f32", seed=3))

    def broken(view):
        raise RuntimeError("peer unreachable")

    with pytest.raises(sa.SinkhornAttnError) as e:
        sa.sinkhorn_attn_fwd_sharded(x["q"], x["k"], x["v"], W=4, eps=1.0, T=2, R=2, halo_lo=0,
                                     halo_hi=0, exchange=broken)
    assert e.value.status == -7
    assert isinstance(e.value.__cause__, RuntimeError)
    torch.cuda.synchronize()  # the context is still usable
