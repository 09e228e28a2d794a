"""The kernels' integer rounding of fp32 to bf16, emulated on the host.

The prefill softmax rounds P to bf16 for the P.V MMA without the conversion
instruction (which shares a unit with the exponentials): it adds 0x8000 to
each fp32 bit pattern and keeps the upper 16 bits (pack_bf16_rna).  That must
equal round-to-nearest of the magnitude with ties away from zero, for every
finite input of either sign: checked here against exact rational rounding."""
import os
import re
from fractions import Fraction

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_io_aware_75_b200", "csrc", "sm100.cuh")


def kernel_pack(lo, hi):
    """The kernel's operations on (lo, hi): two integer adds and a byte
    permute taking bytes 2, 3 of each word (selector 0x7632)."""
    text = open(SRC).read()
    body = re.search(r"uint32_t pack_bf16_rna\(float lo, float hi\) \{(.*?)\n\}", text, re.S)
    assert body, "pack_bf16_rna not found"
    assert "+ 0x8000u" in body.group(1) and "0x7632" in body.group(1)
    a = (np.float32(lo).view(np.uint32).astype(np.uint64) + 0x8000) & 0xFFFFFFFF
    b = (np.float32(hi).view(np.uint32).astype(np.uint64) + 0x8000) & 0xFFFFFFFF
    return int((a >> 16) | ((b >> 16) << 16))


def bf16_value(bits16):
    return float(np.array([bits16 << 16], dtype=np.uint32).view(np.float32)[0])


def rna_reference(x):
    """Exact round-to-nearest (ties away from zero) of float32 x to bf16 bits:
    the nearer of the two bf16 neighbours of x by exact rational distance
    (the one of larger magnitude at a tie)."""
    x = np.float32(x)
    down = int(x.view(np.uint32)) >> 16           # magnitude truncated
    up = down + 1                                  # next magnitude
    xf = Fraction(float(x))
    lo, hi = bf16_value(down), bf16_value(up)
    if not np.isfinite(hi):                        # rounding up overflows: IEEE midpoint rule
        mid = Fraction(float(np.array([(down << 16) | 0x8000], dtype=np.uint32).view(np.float32)[0]))
        return up if abs(xf) >= abs(mid) else down
    return up if abs(Fraction(hi) - xf) <= abs(xf - Fraction(lo)) else down


def test_integer_rounding_is_round_half_away():
    rng = np.random.default_rng(0)
    xs = list(rng.standard_normal(3000).astype(np.float32) * 10)
    xs += list(np.exp2(rng.uniform(-30, 9, 3000)).astype(np.float32))       # softmax weights
    xs += [0.0, -0.0, 1.0, -1.0, 256.0, 2.0 ** -126, -(2.0 ** -126), 3.3895313892515355e38]
    # exact ties and their neighbours
    for base in (1.0, 1.5, 255.0, -3.0, 2.0 ** -20):
        u = int(np.float32(base).view(np.uint32)) & 0xFFFF0000
        for low in (0x7FFF, 0x8000, 0x8001, 0xFFFF):
            xs.append(float(np.array([u | low], dtype=np.uint32).view(np.float32)[0]))
    for i in range(0, len(xs) - 1, 2):
        got = kernel_pack(xs[i], xs[i + 1])
        assert got & 0xFFFF == rna_reference(xs[i]), xs[i]
        assert got >> 16 == rna_reference(xs[i + 1]), xs[i + 1]


def test_agrees_with_round_to_nearest_even_away_from_ties():
    """Off exact ties the result is the hardware conversion's (nearest even)."""
    import torch
    rng = np.random.default_rng(1)
    x = np.exp2(rng.uniform(-20, 8, 20000)).astype(np.float32)
    x = x[(x.view(np.uint32) & 0xFFFF) != 0x8000]
    rne = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    ours = ((x.view(np.uint32).astype(np.uint64) + 0x8000) >> 16).astype(np.uint16)
    assert np.array_equal(rne, ours)
