"""The FMA-pipe 2^x of the softmax, checked directly on the GPU.

Part of each softmax's exponentials bypass the special-function unit: x is
split as n + f with n = round(x), 2^f comes from a degree-3 minimax
polynomial on [-1/2, 1/2] (fitted by csrc/fit_exp2_poly.py, relative error
below 7.5e-5) and 2^n is built in the exponent bits.  End-to-end parity can
hide a 1e-3 error in P under the bf16 output bar, so this test evaluates the
function alone on a dense grid (clamp region, exponent extremes, f = +-1/2
ties) and compares it with the exact 2^x (fp64) and with exp2f (fp32).
"""
import numpy as np
import pytest
import torch

import exact_attention_143_b200 as fa

pytestmark = pytest.mark.gpu

BOUND = 7.5e-5          # the polynomial's fitted relative error
FP32_ROUND = 3 * 2.0 ** -24  # the fp32 Horner and final product add a few roundings


def grid():
    dense = np.linspace(-130.0, 2.0, 1 << 20, dtype=np.float64)
    n = np.arange(-128, 3, dtype=np.float64)
    ties = np.concatenate([n + 0.5, n - 0.5, n, np.nextafter(n + 0.5, -np.inf),
                           np.nextafter(n + 0.5, np.inf)])
    special = np.array([-np.inf, -1e30, -1000.0, -127.0, -126.5, -126.0, -0.0, 0.0, 1.0, 2.0,
                        8.0, 15.5])
    return np.concatenate([dense, ties, special]).astype(np.float32)


@pytest.mark.parametrize("bf16", [False, True], ids=["fp16_kernels", "bf16_kernels"])
def test_fma_exp2_against_exact(bf16):
    x = grid()
    y = fa.selftest_exp2(torch.from_numpy(x).cuda(), bf16=bf16).cpu().numpy().astype(np.float64)
    assert fa.get_device_error() == fa.FA_OK
    xd = x.astype(np.float64)
    exact = np.exp2(xd)
    # from -125.5 up the result is a normal number (n >= -125, or n = -126 with
    # f = +1/2); just below, 2^-126 times p(f) < 1 may be subnormal
    normal = xd >= -125.5
    rel = np.abs(y[normal] / exact[normal] - 1.0)
    assert rel.max() <= BOUND + FP32_ROUND, ("max relative error", rel.max(), xd[normal][rel.argmax()])
    # the bound is close to attained: the polynomial is really the fitted one
    assert rel.max() >= 0.5 * BOUND
    # against the fp32 library function as well
    ref32 = np.exp2(x).astype(np.float64)
    rel32 = np.abs(y[normal] / ref32[normal] - 1.0)
    assert rel32.max() <= BOUND + 2 * FP32_ROUND
    # clamp region: at or below -127 (and -inf, from masked scores) the result is +0
    clamp = xd <= -127.0
    assert np.all(y[clamp] == 0.0) and not np.any(np.signbit(y[clamp]))
    # between -127 and -125.5 the result stays within twice the smallest normal
    tiny = (xd > -127.0) & (xd < -125.5)
    assert np.all(np.abs(y[tiny] - exact[tiny]) <= 2.0 ** -125)
    assert np.all(np.isfinite(y))
