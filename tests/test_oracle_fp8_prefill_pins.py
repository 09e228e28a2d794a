"""Pins for the oracle's FP8 prefill with incoherent processing.

The pages say only that a random orthogonal (Hadamard) transform of Q and K
ahead of FP8 quantisation spreads outliers and lowered the error of FP8
attention 2.6x against plain FP8 (samanvya.dev "Attention Is the Bottleneck",
"FlashAttention: same math, different IO", FlashAttention-3), and that FP8
GEMMs carry a scale per block (Ales Analytics "Attention and matrix kernels",
"How it works").  Pins, none produced by the oracle itself:
  - the rotation against scipy's Hadamard matrix (a library routine) and the
    invariants of an orthogonal map (norms and Q.K dot products kept);
  - E4M3 rounding against torch's float8_e4m3fn cast (a library routine) and
    a brute-force nearest-code search over all 254 finite codes;
  - block scales: the smallest power of two that brings the block's largest
    magnitude to at most 448 (checked against a search over powers of two),
    blocks independent, an all-zero block at scale 1;
  - the attention over codes against the pinned bf16 oracle on values both
    can hold exactly;
  - the pages' claim: with outlier channels the rotated FP8 attention is
    closer to exact attention than FP8 without the rotation.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle


def rnd(shape, seed, std=1.0):
    g = torch.Generator("cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def signs(d, seed):
    return np.where(np.random.default_rng(seed).random(d) < 0.5, -1.0, 1.0)


@pytest.mark.parametrize("d", [8, 64, 128])
def test_rotation_matches_scipy_hadamard(d):
    x = rnd((37, d), d)
    s = signs(d, d + 1)
    ref = (x.double().numpy() * s) @ scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d)
    got = oracle.hadamard_rotate(x, s)
    assert np.abs(got - ref).max() < 1e-13


def test_rotation_keeps_norms_and_dot_products():
    d = 128
    s = signs(d, 3)
    q, k = rnd((64, d), 4), rnd((64, d), 5)
    qr, kr = oracle.hadamard_rotate(q, s), oracle.hadamard_rotate(k, s)
    qd, kd = q.double().numpy(), k.double().numpy()
    assert np.abs(np.linalg.norm(qr, axis=1) - np.linalg.norm(qd, axis=1)).max() < 1e-12
    assert np.abs(qr @ kr.T - qd @ kd.T).max() < 1e-11
    # without signs the map is the identity
    assert np.array_equal(oracle.hadamard_rotate(q, None), qd)


def test_rotation_spreads_an_outlier_channel():
    """A vector with all its mass on one channel comes out flat: |y_c| = |x| / sqrt(d)."""
    d = 64
    x = torch.zeros((1, d), dtype=torch.bfloat16)
    x[0, 17] = 8.0
    y = oracle.hadamard_rotate(x, signs(d, 9))
    assert np.allclose(np.abs(y), 8.0 / math.sqrt(d), rtol=0, atol=1e-15)


def test_e4m3_encode_matches_torch_cast():
    rng = np.random.default_rng(11)
    mag = np.exp2(rng.uniform(-12.0, math.log2(448.0), 20000))
    vals = (mag * np.where(rng.random(20000) < 0.5, -1.0, 1.0)).astype(np.float32)
    # every midpoint between adjacent finite codes (ties) and the codes themselves
    pos = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    mids = (pos[:-1] + pos[1:]) / 2.0
    vals = np.concatenate([vals, pos, -pos, mids, -mids]).astype(np.float32)
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(v)) for v in vals], dtype=np.uint8)
    assert np.array_equal(got, ref)


def test_e4m3_encode_is_nearest_code_ties_to_even():
    codes = [c for c in range(256) if (c & 0x7F) != 0x7F]
    values = np.array([oracle.e4m3_value(c) for c in codes])
    rng = np.random.default_rng(12)
    ys = np.concatenate([rng.uniform(-450, 450, 3000), rng.normal(0, 0.01, 3000)])
    for y in ys:
        got = oracle.e4m3_encode(y)
        dist = np.abs(values - min(max(y, -448.0), 448.0))
        best = [codes[i] for i in np.flatnonzero(dist == dist.min())]
        if len(best) > 1:   # a tie (or +0/-0): the even mantissa, the sign of y
            best = [c for c in best if (c & 1) == 0 and (c >> 7) == (1 if y < 0 else 0)] or best
        assert got in best, (y, got, best)
    # saturation instead of NaN, signed zero kept
    assert oracle.e4m3_encode(1e6) == 0x7E and oracle.e4m3_encode(-1e6) == 0xFE
    assert oracle.e4m3_encode(0.0) == 0x00 and oracle.e4m3_encode(-0.0) == 0x80


def test_block_scales():
    B, N, H, d, blk = 2, 300, 3, 16, 128
    x = np.random.default_rng(13).normal(size=(B, N, H, d))
    x[1, 200:256, 2] = 0.0                     # block 1 of (b=1, h=2) has zeros in part
    x[0, 256:300, 1] = 0.0                     # block 2 of (b=0, h=1): all zero
    x[1, 140, 0, 5] = -37.0                    # an outlier in block 1 of (b=1, h=0)
    codes, scales = oracle.quantize_e4m3_blocks(x, blk)
    assert scales.shape == (B, H, 3)
    for b in range(B):
        for h in range(H):
            for j in range(3):
                xs = x[b, j * blk:(j + 1) * blk, h]
                cs = codes[b, j * blk:(j + 1) * blk, h]
                amax = np.abs(xs).max()
                if amax == 0:
                    assert scales[b, h, j] == 1.0 and np.all(cs == 0)
                    continue
                sc = float(scales[b, h, j])
                # a power of two, the smallest with amax / scale <= 448
                assert sc == 2.0 ** round(math.log2(sc))
                assert amax / sc <= 448.0 < amax / (sc / 2.0)
                # the block's largest magnitude lands in the top binade
                i = np.unravel_index(np.abs(xs).argmax(), xs.shape)
                assert 224.0 <= oracle.e4m3_value(int(cs[i]) & 0x7F) <= 448.0
                # every value within half a grid step (relative 2^-4) of its code
                deq = np.vectorize(oracle.e4m3_value)(cs) * float(scales[b, h, j])
                tol = np.maximum(np.abs(xs) * 2.0 ** -4, 2.0 ** -10 * float(scales[b, h, j]))
                assert np.all(np.abs(deq - xs) <= tol * (1 + 1e-12))
    assert scales[1, 0, 1] == 0.125          # 37 / 0.125 = 296 <= 448 < 592


def test_block_scale_by_search():
    rng = np.random.default_rng(15)
    amaxes = np.concatenate([np.exp2(rng.uniform(-130, 120, 2000)),
                             [448.0, 449.0, 224.0, 223.9, 1.0, 3.5, 7.0, 448.0 * 2 ** -20]])
    for a in amaxes:
        k = -126
        while a / 2.0 ** k > 448.0:
            k += 1
        assert oracle.e4m3_block_scale(a) == np.float32(2.0 ** k), a
    assert oracle.e4m3_block_scale(0.0) == 1.0


@pytest.mark.parametrize("causal,window", [(0, 0), (1, 0), (1, 40)])
def test_attn_fp8_equals_bf16_oracle_on_exact_values(causal, window):
    """Codes times power-of-two scales are bf16 values: both oracles see the same inputs."""
    B, N, Hq, Hkv, d = 2, 150, 4, 2, 32
    rng = np.random.default_rng(14 + causal + window)
    finite = np.array([c for c in range(256) if (c & 0x7F) <= 0x60])   # |value| <= 16
    q8 = rng.choice(finite, (B, N, Hq, d)).astype(np.uint8)
    k8 = rng.choice(finite, (B, N, Hkv, d)).astype(np.uint8)
    v8 = rng.choice(finite, (B, N, Hkv, d)).astype(np.uint8)
    qs = np.exp2(rng.integers(-6, -2, (B, Hq, 2))).astype(np.float32)
    ks = np.exp2(rng.integers(-6, -2, (B, Hkv, 2))).astype(np.float32)
    vs = np.exp2(rng.integers(-3, 2, (B, Hkv))).astype(np.float32)
    table = np.array([oracle.e4m3_value(c) for c in range(256)])
    blk = np.arange(N) // 128
    qv = table[q8] * qs.transpose(0, 2, 1)[:, blk, :, None]
    kv = table[k8] * ks.transpose(0, 2, 1)[:, blk, :, None]
    vv = table[v8] * vs[:, None, :, None]
    as_bf16 = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    assert np.array_equal(as_bf16(qv).double().numpy(), qv)       # exactly representable
    o, lse = oracle.attn_fp8(q8, qs, k8, ks, v8, vs, causal, window, 0.3)
    ro, rl = oracle.attn(as_bf16(qv), as_bf16(kv), as_bf16(vv), causal, window, 0.3)
    assert np.abs(o - ro).max() < 1e-13
    assert np.abs(lse - rl).max() < 1e-13


def test_prepare_layout_and_dequantised_product():
    """fp8_prepare: Q, K rotated then block-quantised; the dequantised Q.K
    products stay within the quantisation error of the exact products."""
    B, N, Hq, Hkv, d = 1, 256, 2, 1, 64
    q, k, v = rnd((B, N, Hq, d), 21), rnd((B, N, Hkv, d), 22), rnd((B, N, Hkv, d), 23)
    s = signs(d, 24)
    p = oracle.fp8_prepare(q, k, v, s)
    assert p["q8"].shape == (B, N, Hq, d) and p["q_scale"].shape == (B, Hq, 2)
    assert p["k_scale"].shape == (B, Hkv, 2) and p["v_scale"].shape == (B, Hkv)
    table = np.array([oracle.e4m3_value(c) for c in range(256)])
    vdeq = table[p["v8"]] * p["v_scale"][:, None, :, None]
    assert np.abs(vdeq - v.double().numpy()).max() <= 2.0 ** -4 * np.abs(v.double().numpy()).max()
    qdeq = table[p["q8"][0, :, 0]] * np.repeat(p["q_scale"][0, 0], 128)[:, None]
    kdeq = table[p["k8"][0, :, 0]] * np.repeat(p["k_scale"][0, 0], 128)[:, None]
    exact = q[0, :, 0].double().numpy() @ k[0, :, 0].double().numpy().T
    rel = np.abs(qdeq @ kdeq.T - exact).max() / np.abs(exact).max()
    assert rel < 0.05


def test_incoherent_processing_reduces_error_with_outliers():
    """The pages' claim: with outlier channels in Q and K, rotating before
    quantisation brings FP8 attention closer to exact attention (they report
    2.6x lower error); here at least 2x lower RMS error on O."""
    B, N, Hq, Hkv, d = 1, 384, 4, 2, 128

    def with_outliers(H, seed):
        x = torch.randn((B, N, H, d), generator=torch.Generator().manual_seed(seed))
        x[..., [3, 77, 100]] *= 20.0
        return x.to(torch.bfloat16)

    q, k = with_outliers(Hq, 31), with_outliers(Hkv, 32)
    v = rnd((B, N, Hkv, d), 33)
    sc = 0.1 / math.sqrt(d)
    ref, _ = oracle.attn(q, k, v, True, 0, sc)
    o_plain, _, _ = oracle.fp8_prefill(q, k, v, None, causal=True, scale=sc)
    o_rot, _, _ = oracle.fp8_prefill(q, k, v, signs(d, 34), causal=True, scale=sc)
    e_plain = np.sqrt(((o_plain - ref) ** 2).mean())
    e_rot = np.sqrt(((o_rot - ref) ** 2).mean())
    assert e_rot * 2.0 < e_plain, (e_rot, e_plain)


def test_attn_fp8_rows_are_a_selection():
    B, N, Hq, Hkv, d = 2, 200, 2, 1, 16
    rng = np.random.default_rng(41)
    finite = np.array([c for c in range(256) if (c & 0x7F) <= 0x58])
    q8 = rng.choice(finite, (B, N, Hq, d)).astype(np.uint8)
    k8 = rng.choice(finite, (B, N, Hkv, d)).astype(np.uint8)
    v8 = rng.choice(finite, (B, N, Hkv, d)).astype(np.uint8)
    qs = rng.uniform(0.01, 0.1, (B, Hq, 2)).astype(np.float32)
    ks = rng.uniform(0.01, 0.1, (B, Hkv, 2)).astype(np.float32)
    vs = rng.uniform(0.5, 2.0, (B, Hkv)).astype(np.float32)
    rows = [0, 5, 127, 128, 199]
    for causal, window in ((0, 0), (1, 0), (1, 30)):
        o, lse = oracle.attn_fp8(q8, qs, k8, ks, v8, vs, causal, window, 0.2)
        os_, ls = oracle.attn_fp8(q8, qs, k8, ks, v8, vs, causal, window, 0.2, rows=rows)
        assert np.array_equal(os_, o[:, rows]) and np.array_equal(ls, lse[:, :, rows])
