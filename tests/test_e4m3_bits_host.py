"""Host check of the FP8 decode kernel's E4M3 -> fp32 conversion by bit
placement (decode_sm100.cu, e4m3x4_to_f32): for every code in every byte
position of a 32-bit word, the fp32 it builds times 2^120 is the code's
value (torch's float8_e4m3fn, a library decoder), the other three outputs
are +0, and signs and subnormal codes come out exact."""
import math
import struct

import torch


def f32(bits):
    return struct.unpack("<f", struct.pack("<I", bits & 0xFFFFFFFF))[0]


def kernel_formula(w):
    """The four fp32 values e4m3x4_to_f32 produces for word w, in code order."""
    h = ((w & 0x7F007F00) >> 4) | (w & 0x80008000)
    g = ((w & 0x007F007F) << 4) | ((w << 8) & 0x80008000)
    return [f32(g << 16), f32(h << 16), f32(g & 0xFFFF0000), f32(h & 0xFFFF0000)]


def test_every_code_every_position():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().tolist()
    for c in range(256):
        if math.isnan(ref[c]):
            continue
        for pos in range(4):
            vals = kernel_formula(c << (8 * pos))
            v = vals[pos] * 2.0 ** 120
            assert v == ref[c] and math.copysign(1, v) == math.copysign(1, ref[c]), (c, pos)
            assert all(vals[q] == 0.0 for q in range(4) if q != pos)


def test_mixed_word():
    codes = [0x38, 0xB8, 0x01, 0x7E]          # 1, -1, 2^-9, 448
    w = sum(c << (8 * i) for i, c in enumerate(codes))
    got = [x * 2.0 ** 120 for x in kernel_formula(w)]
    assert got == [1.0, -1.0, 2.0 ** -9, 448.0]
