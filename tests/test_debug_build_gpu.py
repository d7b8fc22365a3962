"""The debug build (-DSA_DEBUG, libsinkhorn_attn_debug.so): every kernel checks
the indices of its guarded accesses and records SA_ERR_BOUNDS instead of
trapping.  On the small parity cases (both storage types, masks, the dustbin,
W = 0 and dense W, several tail lengths, more tiles than persistent CTAs) the
checked library must report no failed check and still match the oracle.  It
runs in a child process so that only the debug library is loaded there."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r"""
import sys
sys.path.insert(0, ROOT)
import torch
import banded_log_domain_b200 as sa
from tests import parity
assert sa.LIB_PATH.endswith("libsinkhorn_attn_debug.so"), sa.LIB_PATH
CASES = [
    # (L, W, eps, T, R, dtype, mask_kind/valid_len, dustbin)
    (17, 5, 0.8, 3, 2, "f32", None, False),
    (200, 17, 0.6, 4, 3, "f32", "holes", False),
    (160, 20, 0.7, 4, 2, "f32", "holes", True),
    (64, 0, 1.0, 2, 2, "bf16", None, False),
    (100, 150, 1.0, 2, 2, "bf16", "holes", False),
    (520, 64, 0.6, 4, 3, "bf16", "holes", False),
    (700, 256, 1.0, 2, 4, "bf16", None, False),
    (300, 100, 1.0, 2, 9, "bf16", (180, 300), False),
    (8192, 64, 0.9, 3, 2, "bf16", (6000, 8192), False),
]
for case in CASES:
    L, W, eps, T, R, dtype, mk, db = case
    B, H = 2, 2
    x = parity.draw_case(B, H, L, dtype=dtype, seed=L + 31 * W,
                         mask_kind=mk if isinstance(mk, str) else None,
                         valid_len=mk if isinstance(mk, tuple) else None, dustbin=db,
                         v_dust_random=db)
    d = parity.to_dev(x)
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    p = sa.make_params(B, H, L, 64, W=W, eps=eps, T=T, R=R, dtype=td, dustbin=db, dustbin_score=-1.2)
    fws, bws = sa.sinkhorn_attn_workspace_size(p)
    wsf = torch.zeros(fws, dtype=torch.uint8, device="cuda")
    kw = dict(W=W, eps=eps, R=R, mask=d["mask"], dustbin=db, dustbin_score=-1.2, v_dust=d["v_dust"])
    o, st = sa.sinkhorn_attn_fwd(d["q"], d["k"], d["v"], T=T, ws=wsf, **kw)
    assert sa.sinkhorn_attn_poll(wsf) == 0, ("forward status", case)
    g = {"o": o, "state": st}
    for sched in ("one_reference", "direct"):
        wsb = torch.zeros(bws, dtype=torch.uint8, device="cuda")
        dsc = torch.zeros(1, device="cuda") if db else None
        out = sa.sinkhorn_attn_bwd(d["q"], d["k"], d["v"], o, d["dO"], st, schedule=sched, ws=wsb,
                                   d_dust_score=dsc, **kw)
        assert sa.sinkhorn_attn_poll(wsb) == 0, ("backward status", sched, case)
        g[sched] = tuple(out) + (dsc,)
    torch.cuda.synchronize()
    to = lambda t: None if t is None else (tuple(to(u) for u in t) if isinstance(t, tuple)
                                           else t.detach().float().cpu().double().numpy())
    g = {k: to(v) for k, v in g.items()}
    r = parity.oracle_run(x, W=W, eps=eps, T=T, R=R, dustbin=db, dustbin_score=-1.2)
    parity.compare(x, g, r, dtype=dtype, dustbin=db, schedules=("one_reference", "direct"),
                   label="debug build " + str(case))
print("DEBUG-BUILD-OK")
"""


def test_debug_build_reports_no_bounds_failure_and_matches_the_oracle():
    import banded_log_domain_b200 as sa

    assert os.path.exists(sa.DEBUG_LIB_PATH), "build the debug library first"
    env = dict(os.environ, SINKHORN_ATTN_DEBUG_LIB="1")
    r = subprocess.run([sys.executable, "-c", "ROOT = %r\n" % ROOT + CHILD], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "DEBUG-BUILD-OK" in r.stdout, (r.stdout[-2000:], r.stderr[-4000:])
