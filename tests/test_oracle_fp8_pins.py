"""Pins for the oracle's FP8 (E4M3) paged-cache decode.

The post names an FP8 KV cache as a routine option (samanvya.dev "Attention
Is the Bottleneck", the cache-size paragraphs before "Paging and prefix
sharing") without fixing a format; the reading taken is OCP FP8 E4M3 ("fn":
no infinities) with one fp32 scale per (page, KV head).  Pins, none produced
by the oracle:
  - every one of the 256 codes decodes to torch's float8_e4m3fn value (a
    library routine), and a few codes worked by hand from the format;
  - with power-of-two scales the dequantised values are exactly bf16, and the
    FP8 decode equals the (pinned) bf16 decode on that cache bit for bit;
  - a power-of-two factor moved from the K scales into q changes nothing.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads


def test_all_codes_match_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x80, -0.0), (0x38, 1.0), (0xB8, -1.0), (0x7E, 448.0), (0x01, 2.0 ** -9),
    (0x08, 2.0 ** -6), (0x07, 7 * 2.0 ** -9), (0x40, 2.0), (0x3C, 1.5)])
def test_hand_codes(code, value):
    got = oracle.e4m3_value(code)
    assert got == value and math.copysign(1, got) == math.copysign(1, value)
    assert math.isnan(oracle.e4m3_value(0x7F)) and math.isnan(oracle.e4m3_value(0xFF))


def dequant_bf16(codes, scale):
    v = codes.view(torch.float8_e4m3fn).double() * scale.double()[:, None, :, None]
    b = v.to(torch.bfloat16)
    assert torch.equal(b.double(), v) or torch.isnan(v).any()   # exact with pow2 scales
    return b


@pytest.mark.parametrize("sinks", [False, True])
def test_pow2_scales_equal_bf16_decode(sinks):
    w = workloads.paged_fp8(pow2_scales=True, lens=[1, 16, 37, 300], Hq=8, Hkv=2, d=64,
                            seed=3)
    kb, vb = dequant_bf16(w.k_codes, w.k_scale), dequant_bf16(w.v_codes, w.v_scale)
    z = np.array([0.5, -1.0, -math.inf, 2.0, 0.0, 1.0, -3.0, 4.0]) if sinks else None
    o8, l8 = oracle.decode_paged_fp8(w.q, w.k_codes, w.v_codes, w.k_scale, w.v_scale,
                                     w.block_table, w.seq_lens, w.scale, sinks=z)
    if sinks:
        ob, lb = oracle.decode_paged_sinks(w.q, kb, vb, w.block_table, w.seq_lens, z, w.scale)
    else:
        ob, lb = oracle.decode_paged(w.q, kb, vb, w.block_table, w.seq_lens, w.scale)
    assert np.array_equal(o8, ob) and np.array_equal(l8, lb)


def test_scale_moves_between_q_and_k():
    w = workloads.paged_fp8(lens=[50, 129], Hq=4, Hkv=2, d=64, seed=5)
    o1, l1 = oracle.decode_paged_fp8(w.q, w.k_codes, w.v_codes, w.k_scale, w.v_scale,
                                     w.block_table, w.seq_lens, w.scale)
    q2 = (w.q.double() * 0.5).to(torch.bfloat16)
    assert torch.equal(q2.double(), w.q.double() * 0.5)
    o2, l2 = oracle.decode_paged_fp8(q2, w.k_codes, w.v_codes, w.k_scale * 2, w.v_scale,
                                     w.block_table, w.seq_lens, w.scale)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)
