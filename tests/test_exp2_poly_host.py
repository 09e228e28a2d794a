"""The prefill kernel's software exponential, emulated on the host in fp32.

The kernel computes 2^x for part of the scores on the FMA pipe: x = j + f
with j = floor(x), 2^f from a cubic, 2^j added into the exponent bits
("FlashAttention-4": software exponentials).  These checks read the cubic's
coefficients out of the kernel source and pin the evaluation against numpy's
exp2 over the range the kernel uses; P is then rounded to bf16 (relative
2^-9), so the cubic must be far more accurate than that."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_io_aware_75_b200", "csrc", "sm100.cuh")


def coefficients():
    text = open(SRC).read()
    m = re.search(r"constexpr float c1 = ([0-9.e+-]+)f, c2 = ([0-9.e+-]+)f, c3 = ([0-9.e+-]+)f;",
                  text)
    assert m, "coefficients not found"
    return [np.float32(1.0)] + [np.float32(float(g)) for g in m.groups()]


def kernel_exp2(x):
    """The kernel's sequence of fp32 operations, one by one."""
    c = coefficients()
    x = np.maximum(x.astype(np.float32), np.float32(-127.0))
    shift = np.float32(12582912.0)
    # round-down add: floor(x) lands in the low mantissa bits
    y = (np.floor(x.astype(np.float64)) + 12582912.0).astype(np.float32)
    j = (y - shift).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (np.float32(c[3]) * f + c[2]).astype(np.float32)
    p = (p * f + c[1]).astype(np.float32)
    p = (p * f + c[0]).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + (y.view(np.uint32).astype(np.uint64) << 23))
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_relative_error_over_range():
    x = np.linspace(-126.0, 8.0, 1_000_001, dtype=np.float64).astype(np.float32)
    got = kernel_exp2(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 1.0e-4            # bf16 rounding of P is 2^-9 ~ 2e-3


def test_exact_at_integers_and_zero():
    for k in range(-20, 9):
        assert kernel_exp2(np.array([k], np.float32))[0] == np.float32(2.0 ** k)


def test_masked_scores_vanish():
    tiny = kernel_exp2(np.array([-np.inf, -1e30, -200.0, -127.0], np.float32))
    assert np.all(tiny >= 0) and np.all(tiny < 2.0 ** -125)


def test_monotone_on_grid():
    x = np.linspace(-30.0, 8.0, 200_001).astype(np.float32)
    y = kernel_exp2(x)
    assert np.all(np.diff(y.astype(np.float64)) >= 0)
