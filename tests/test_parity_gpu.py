"""GPU (C ABI, CUDA kernels) vs the CPU oracle on the same seeded inputs.

Small cases cover several row blocks and a ragged tail, the edge cases of the
method (L = 1, W = 0, dense W >= L, T = 0, R = 1..20, masks with holes, fully
padded sequences, the dustbin), both storage types and both backward
schedules.  The named workloads run at their full sizes; the two largest are
compared on a subset of heads (every (batch, head) problem is independent).
"""
import numpy as np
import pytest

import workloads
from tests import parity

pytestmark = pytest.mark.gpu

SMALL = [
    # (L, W, eps, T, R, dtype, mask_kind/valid_len, dustbin)
    (1, 3, 1.0, 2, 2, "f32", None, False),
    (2, 1, 0.7, 1, 2, "f32", None, False),
    (3, 0, 0.5, 2, 2, "f32", None, False),
    (17, 5, 0.8, 3, 2, "f32", None, False),
    (64, 63, 1.0, 2, 2, "f32", None, False),
    (65, 64, 1.0, 2, 2, "f32", "holes", False),
    (130, 5, 0.5, 0, 2, "f32", None, False),
    (130, 200, 1.0, 3, 2, "f32", "holes", False),
    (200, 17, 0.6, 4, 1, "f32", (100, 200), False),
    (200, 17, 0.6, 4, 3, "f32", "holes", False),
    (150, 9, 0.9, 2, 4, "f32", None, False),
    (190, 33, 1.0, 5, 2, "bf16", (90, 190), False),
    (100, 7, 1.0, 3, 2, "f32", None, True),
    (160, 20, 0.7, 4, 2, "f32", "holes", True),
    (140, 11, 1.0, 2, 2, "bf16", None, True),
    (129, 1, 1.0, 3, 2, "bf16", "holes", False),
    # tensor-core path (bf16, no dustbin): tiles of 128 rows x 128-column chunks
    (17, 5, 0.8, 3, 2, "bf16", None, False),
    (64, 0, 1.0, 2, 2, "bf16", None, False),
    (100, 150, 1.0, 2, 2, "bf16", "holes", False),
    (300, 200, 0.7, 0, 2, "bf16", None, False),
    (384, 128, 1.0, 3, 1, "bf16", (200, 384), False),
    (520, 64, 0.6, 4, 3, "bf16", "holes", False),
    (700, 256, 1.0, 2, 4, "bf16", None, False),
    (1000, 37, 0.9, 5, 2, "bf16", (600, 1000), False),
    # tails longer than one dS sweep's 8 modifier terms: 2, 3 and 5 blocks of
    # terms summed in fp32; T = 0 with R = N is full backpropagation
    (150, 9, 0.9, 0, 5, "f32", None, False),
    (130, 7, 1.0, 1, 9, "f32", "holes", True),
    (520, 64, 0.6, 0, 5, "bf16", "holes", False),
    (300, 100, 1.0, 2, 9, "bf16", (180, 300), False),
    (384, 64, 1.0, 0, 20, "bf16", None, False),
    # more tiles than the 148 persistent CTAs (2 x 2 problems x 64 row blocks):
    # CTAs walk several tiles, and the dS sweeps read a tile's rows out of TMEM
    # after the next tile's first chunk
    (8192, 64, 0.9, 3, 2, "bf16", (6000, 8192), False),
    (8192, 100, 1.0, 2, 1, "bf16", "holes", False),
    # every chunk count modulo the four epilogue parts (a chunk's readers then
    # fall on different parts): 2W + 128 over 128 = 4, 6, 7
    (4096, 192, 1.0, 3, 2, "bf16", "holes", False),
    (4096, 320, 0.8, 2, 2, "bf16", None, False),
    (4096, 384, 1.0, 2, 1, "bf16", (3000, 4096), False),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "L{}_W{}_T{}_R{}_{}_{}_{}".format(
    c[0], c[1], c[3], c[4], c[5], c[6], "db" if c[7] else "nodb"))
def test_small_cases(case):
    L, W, eps, T, R, dtype, mk, db = case
    B, H = 2, 2
    x = parity.draw_case(B, H, L, dtype=dtype, seed=L + 31 * W,
                         mask_kind=mk if isinstance(mk, str) else None,
                         valid_len=mk if isinstance(mk, tuple) else None, dustbin=db,
                         v_dust_random=db)
    kw = dict(W=W, eps=eps, T=T, R=R, dustbin=db, dustbin_score=-1.2)
    plans = [(R, R), (R, R - 1)] + ([(1, 0)] if R >= 1 else [])
    g = parity.gpu_run(x, schedules=("one_reference", "direct"), plans=plans, **kw)
    r = parity.oracle_run(x, plans=plans, **kw)
    parity.compare(x, g, r, dtype=dtype, dustbin=db, schedules=("one_reference", "direct"),
                   label=str(case))
    parity.compare_plans(g, r, plans, dtype=dtype, label=str(case))


def test_fully_padded_sequence_is_zero():
    x = parity.draw_case(2, 1, 80, seed=5, valid_len=(40, 80))
    x["mask"][1] = 0
    kw = dict(W=6, eps=0.7, T=3, R=2)
    g = parity.gpu_run(x, schedules=("one_reference", "direct"), **kw)
    r = parity.oracle_run(x, **kw)
    parity.compare(x, g, r, dtype="f32", dustbin=False, schedules=("one_reference", "direct"))
    assert np.all(g["o"][1] == 0) and np.all(g["state"][1] == 0)


def _named(name, heads=None):
    w, x = workloads.make(name)
    kw = dict(W=w.W, eps=w.eps, T=w.T, R=w.R, dustbin=w.dustbin, dustbin_score=w.dustbin_score)
    g = parity.gpu_run(x, schedules=("one_reference", "direct"), plans=[(2, 2)], **kw)
    r = parity.oracle_run(x, plans=[(2, 2)], heads=heads, **kw)
    parity.compare(x, g, r, dtype=w.dtype, dustbin=w.dustbin, heads=heads,
                   schedules=("one_reference", "direct"), label=name)
    parity.compare_plans(g, r, [(2, 2)], dtype=w.dtype, heads=heads, label=name)


def test_workload_small512():
    _named("small512")


def test_workload_masked2k():
    _named("masked2k")


def test_workload_dustbin4k():
    _named("dustbin4k")


@pytest.mark.slow
def test_workload_long32k_sampled_heads():
    """Full-size long-context workload through the same calls the benchmark
    times; two heads compared with the oracle in full."""
    w, x = workloads.make("long32k")
    heads = [0, 11]
    kw = dict(W=w.W, eps=w.eps, T=w.T, R=w.R)
    g = parity.gpu_run(x, schedules=("one_reference",), **kw)
    r = parity.oracle_run(x, heads=heads, **kw)
    parity.compare(x, g, r, dtype=w.dtype, dustbin=False, heads=heads, label="long32k")


@pytest.mark.slow
def test_workload_vjp262k_windows():
    """L = 262144: the GPU runs the whole sequence; the oracle runs windows of
    it.  A token's outputs and gradients depend only on tokens within
    (2(T+R) + 7) W of it (each half-sweep widens the dependence by W), so on a
    window the oracle is exact away from the cut ends."""
    w, x = workloads.make("vjp262k")
    kw = dict(W=w.W, eps=w.eps, T=w.T, R=w.R)
    g = parity.gpu_run(x, schedules=("one_reference", "direct"), **kw)
    reach = (2 * (w.T + w.R) + 7) * w.W
    L = w.L
    for lo, hi in ((0, 2 * reach + 2048), (L // 2 - reach - 1024, L // 2 + reach + 1024),
                   (L - 2 * reach - 2048, L)):
        sub = {k: (None if v is None else (v[:, :, lo:hi] if v.dim() == 4 else v))
               for k, v in x.items()}
        r = parity.oracle_run(sub, heads=[3], **kw)
        keep_lo = lo if lo == 0 else lo + reach
        keep_hi = hi if hi == L else hi - reach
        rows = slice(keep_lo - lo, keep_hi - lo)
        gsub = {"o": g["o"][:, :, lo:hi], "state": g["state"][..., lo:hi]}
        for s in ("one_reference", "direct"):
            gsub[s] = tuple(None if t is None else t[:, :, lo:hi] for t in g[s])
        parity.compare(sub, gsub, r, dtype=w.dtype, dustbin=False, heads=[3], rows=rows,
                       schedules=("one_reference", "direct"), label=f"vjp262k[{lo}:{hi}]")
