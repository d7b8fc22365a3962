"""The exponentials of the row-sum sweeps (dual updates and vector-cotangent
sweeps): part of every 32 in-band entries is evaluated on the FMA pipe by
range reduction and a fitted polynomial, the rest by ex2.approx on the MUFU
unit.  Both must agree with 2^x in double precision to the accuracy the
sweeps rely on (a few units in the last place of float32)."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def test_polynomial_exp2_matches_exact_and_mufu():
    import banded_log_domain_b200 as sa

    g = torch.Generator().manual_seed(0)
    dense = torch.linspace(-126.0, 0.0, 2_000_001)
    rnd = -torch.rand(1_000_000, generator=g) * 40.0
    # around the reduction's cut points n +- 1/2 and small magnitudes
    cuts = torch.arange(-126, 1, dtype=torch.float32)[:, None] + torch.tensor(
        [-0.5, -0.4999999, 0.5, 0.4999999, -1e-7, 1e-7])[None, :]
    x = torch.cat([dense, rnd, cuts.flatten().clamp(max=0.0), torch.tensor([0.0, -0.0])])
    x = x.contiguous().cuda()
    yp, ym = sa.sinkhorn_attn_debug_exp2(x)
    torch.cuda.synchronize()
    xd = x.double().cpu().numpy()
    exact = np.exp2(xd)
    rp = np.abs(yp.double().cpu().numpy() / exact - 1.0)
    rm = np.abs(ym.double().cpu().numpy() / exact - 1.0)
    # normal results (x >= -125): a relative error of a few float32 ulps
    nrm = xd >= -125.0
    assert rp[nrm].max() <= 4.0e-7, rp[nrm].max()
    assert rm[nrm].max() <= 4.0e-7, rm[nrm].max()
    assert np.sqrt((rp[nrm] ** 2).mean()) <= 1.5e-7
    # the bottom of the range: tiny and non-negative, never above 2^-124
    low = yp.double().cpu().numpy()[~nrm]
    assert (low >= 0).all() and (low <= 2.0 ** -124).all()
    # x = 0 is exactly 1 within one ulp
    assert abs(float(yp[-1]) - 1.0) <= 2.0 ** -23


def test_polynomial_exp2_clamps_minus_infinity():
    import banded_log_domain_b200 as sa

    x = torch.tensor([-float("inf"), -1000.0, -127.0, -126.0], device="cuda")
    yp, ym = sa.sinkhorn_attn_debug_exp2(x)
    torch.cuda.synchronize()
    assert (yp.cpu() >= 0).all() and (yp.cpu() <= 2.0 ** -124).all()
    assert float(ym[0]) == 0.0
