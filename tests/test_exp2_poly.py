"""The FMA-pipe exponential the forward kernel can use for part of its
probabilities (switched off in this build, FWD_POLY_PERIOD = 0): fitted
coefficients (CPU) and the device implementation against torch.exp2 (GPU)."""
import os
import re

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HDR = os.path.join(ROOT, "exact_tiled_attention_46_b200", "csrc", "exp2_poly.cuh")


def coefficients():
    txt = open(HDR).read()
    deg = int(re.search(r"FA_EXP2_POLY_DEGREE (\d+)", txt).group(1))
    c = [float(re.search(rf"FA_EXP2_C{i} ([-0-9.e]+)f", txt).group(1)) for i in range(deg + 1)]
    bound = float(re.search(r"#define FA_EXP2_MAX_REL_ERR ([-0-9.e]+)", txt).group(1))
    return np.array(c, dtype=np.float32), bound


def test_fitted_polynomial_meets_its_bound_and_bf16_needs():
    c, bound = coefficients()
    f = np.linspace(-0.5, 0.5, 100001)
    p = np.zeros_like(f)
    for a in c[::-1].astype(np.float64):
        p = p * f + a
    err = np.max(np.abs(p / np.exp2(f) - 1))
    assert err <= bound * 1.001
    assert bound < 2.0 ** -12          # far below half the bf16 spacing (2^-9)


@pytest.mark.gpu
def test_device_exp2_poly_vs_torch():
    from parity import need_gpu
    need_gpu()
    import exact_tiled_attention_46_b200 as fa
    _, bound = coefficients()
    # relative accuracy holds where 2^x is a normal float with margin (x >= -125);
    # below, the results only have to be negligibly small
    x = torch.cat([torch.linspace(-125.0, 16.0, 1 << 20), torch.tensor([0.0, -0.5, 0.5, 15.75, -124.5]),
                   torch.tensor([-126.0, -200.0, float("-inf")]),
                   torch.tensor([128.0, 130.5, 1000.0, float("inf")])])
    x = x.to(torch.float32).cuda()
    y = torch.empty_like(x)
    assert fa.lib().fa_selftest_exp2_poly(x.data_ptr(), y.data_ptr(), x.numel(),
                                          torch.cuda.current_stream().cuda_stream) == fa.FA_OK
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    ok = (x >= -125.0) & (x <= 127.0)
    rel = ((y.double() - ref) / ref).abs()[ok]
    assert float(rel.max()) <= bound + 2.0 ** -20
    tiny = y[~ok & (x < 0)]
    assert torch.all(tiny >= 0) and torch.all(tiny < 2.0 ** -125)
    # above the clamp the result stays the finite 2^127 (a large positive
    # number that trips the fast path's sum limit), never a wrapped exponent
    big = y[x > 127.0]
    assert big.numel() == 4 and torch.all(torch.isfinite(big)) and torch.all(big > 2.0 ** 126)
