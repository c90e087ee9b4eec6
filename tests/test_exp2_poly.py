"""The FMA-pipe exponential of the forward kernels.

A share of the softmax weights 2^(s - m) ("FlashAttention" explainer page, How
it works, Step 3) is computed on the FMA pipe instead of the MUFU unit: with
n = rint(x) and f = x - n, 2^f comes from a cubic fitted for minimax relative
error on [-1/2, 1/2] (Cody-Waite style reduction; Lawson iterations), and 2^n is
built in the exponent field.

CPU: re-running the committed generator reproduces the committed coefficients
and error bound.  GPU (through the C ABI self-test entry point): a dense grid and
the edge cases against 2^x in float64 -- the relative error stays within the
generator's bound where 2^x is a normal float, integer arguments give exact
powers of two, and arguments below -126.5 (a masked key's -inf among them) give
exactly 0."""
from __future__ import annotations

import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "exact_attention_142_b200", "csrc", "exp2_poly.cuh")


def committed():
    text = open(HEADER).read()
    vals = dict(re.findall(r"constexpr float (k\w+) = ([-+0-9.eE]+)f;", text))
    return ([float(vals["kC1"]), float(vals["kC2"]), float(vals["kC3"])],
            float(vals["kMaxRelError"]))


def test_generator_reproduces_the_committed_polynomial():
    from exact_attention_142_b200.csrc import gen_exp2_poly as gen
    coeffs, bound = committed()
    fitted = gen.fit()
    for c_fit, c_com in zip(fitted, coeffs):
        # the committed values are the float32 roundings of the fit
        assert abs(float(np.float32(c_fit)) - c_com) <= 2 * np.spacing(np.float32(c_com)), (c_fit, c_com)
    err = gen.max_rel_error_f32(coeffs)
    assert abs(err - bound) <= 1e-9, (err, bound)
    # a cubic on [-1/2, 1/2]: the minimax relative error of 2^f is about 1e-4,
    # well below the bf16 rounding of the weights (2^-9)
    assert 5e-5 < bound < 2e-4


def test_committed_polynomial_is_near_minimax():
    """Equal ripple: with three free coefficients (the constant term is pinned
    to 1, which forces a zero of the error at f = 0), a minimax fit reaches its
    maximum relative error at no fewer than four points of the interval."""
    coeffs, _ = committed()
    f = np.linspace(-0.5, 0.5, 200001)
    p = 1 + coeffs[0] * f + coeffs[1] * f ** 2 + coeffs[2] * f ** 3
    r = p / np.exp2(f) - 1
    emax = np.abs(r).max()
    peaks = [i for i in range(1, len(f) - 1) if abs(r[i]) >= abs(r[i - 1]) and abs(r[i]) >= abs(r[i + 1])]
    peaks = [0] + peaks + [len(f) - 1]
    assert sum(1 for i in peaks if abs(r[i]) > 0.99 * emax) >= 4
    assert r[np.argmin(np.abs(f))] == pytest.approx(0.0, abs=1e-12)  # 2^0 = 1 exactly


@pytest.mark.gpu
def test_exp2_poly_on_the_gpu():
    import torch

    import exact_attention_142_b200 as ea
    from exact_attention_142_b200 import build
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    _, bound = committed()
    grid = np.linspace(-130.0, 8.0, 552001).astype(np.float32)
    ints = np.arange(-130, 9).astype(np.float32)
    edges = np.array([0.0, -0.0, 0.5, -0.5, 0.25, -0.25, 1e-7, -1e-7, 7.999, 8.0, -1.5, -2.5,
                      -124.5, -125.0, -125.5, -125.75, -126.0, -126.25, -126.5, -126.5001,
                      -126.75, -127.0, -127.5, -128.0, -150.0, -1e30, -np.inf],
                     dtype=np.float32)
    x = np.concatenate([grid, ints, edges, np.nextafter(edges, np.float32(-np.inf))])
    xd = torch.from_numpy(x).cuda()
    yd = torch.full_like(xd, float("nan"))
    ea.attn_selftest_exp2_poly(xd, yd, xd.numel())
    torch.cuda.synchronize()
    y = yd.cpu().numpy().astype(np.float64)
    xf = x.astype(np.float64)
    ref = np.exp2(xf)
    assert np.isfinite(y).all() and (y >= 0).all()
    # below the clamp: exactly zero (-inf, the masked keys, among them)
    low = xf < -126.5
    assert (y[low] == 0.0).all(), x[low][y[low] != 0.0][:8]
    # normal results: the generator's relative bound (plus a few fp32 roundings
    # of the fused evaluation, which the generator models unfused)
    normal = ref >= 2.0 ** -126
    rel = np.abs(y[normal] / ref[normal] - 1.0)
    assert rel.max() <= bound + 2.0 ** -21, (rel.max(), bound)
    # between: subnormal results, within the bound or one subnormal spacing
    mid = ~low & ~normal
    assert (np.abs(y[mid] - ref[mid]) <= bound * ref[mid] + 2.0 ** -148).all()
    # integers: f = 0 and 2^0 = 1, so the result is the exact power of two
    isint = (xf == np.round(xf)) & (xf >= -126) & (xf <= 8)
    assert (y[isint] == ref[isint]).all()
