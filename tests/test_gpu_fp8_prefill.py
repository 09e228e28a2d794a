"""GPU parity of the FP8 prefill (fa_fp8_prepare + fa_fwd_fp8) against the
fp64 oracle's FP8 prefill, through the C ABI.

* fa_fp8_prepare: scales and E4M3 codes against the oracle's rotation and
  quantisation (codes equal except at near-ties, see parity.compare_codes),
  V's codes in the transposed layout.
* fa_fwd_fp8 on the oracle's own codes: within the FP8 bound of
  parity.compare_fp8 of the oracle's attention over those codes; LSE within
  the bf16 tolerance.  The padding bytes of V^T are poisoned with NaN codes.
* The two calls end to end, and the pages' claim (rotation lowers FP8 error
  when Q and K have outlier channels) on the GPU's results.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import code_flip_score_bound, compare_codes, compare_fp8, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_io_aware_75_b200 as fa
    return fa


def signs(d, seed):
    return np.where(np.random.default_rng(seed).random(d) < 0.5, -1.0, 1.0)


def inputs(B, N, Hq, Hkv, seed, outliers=False):
    inp = workloads.dense(B, Hq, Hkv, N, 128, causal=True, seed=seed)
    q, k, v = inp.q, inp.k, inp.v
    if outliers:
        q, k = q.float(), k.float()
        q[..., [3, 77, 100]] *= 20.0
        k[..., [3, 77, 100]] *= 20.0
        q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    return q, k, v


def to_device_prep(p, N):
    """The oracle's operands in the library's layouts; V^T padding = NaN codes."""
    B, _, Hkv, d = p["v8"].shape
    vts = (N + 15) // 16 * 16
    vt = np.full((B, Hkv, d, vts), 0x7F, np.uint8)
    vt[..., :N] = p["v8"].transpose(0, 2, 3, 1)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return {"q8": dev(p["q8"]), "k8": dev(p["k8"]), "vt8": dev(vt),
            "q_scale": dev(p["q_scale"]), "k_scale": dev(p["k_scale"]),
            "v_scale": dev(p["v_scale"])}


def abs_v(p):
    return np.bitwise_and(p["v8"], 0x7F)


@pytest.mark.parametrize("B,N,Hq,Hkv,rot", [
    (1, 128, 2, 1, True), (2, 300, 4, 2, True), (1, 77, 4, 4, False), (1, 1000, 8, 2, True)])
def test_prepare_matches_oracle(fa, B, N, Hq, Hkv, rot):
    q, k, v = inputs(B, N, Hq, Hkv, seed=N + Hq)
    s = signs(128, N) if rot else None
    ref = oracle.fp8_prepare(q, k, v, s)
    sg = torch.tensor(s, dtype=torch.float32).cuda() if rot else None
    got = fa.fp8_prepare(q.cuda(), k.cuda(), v.cuda(), sg)
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    # Power-of-two scales: equal on both sides.  Codes of exact inputs (V, and
    # Q, K without the rotation) are decided on the same exact values: equal
    # bit for bit; rotated Q, K come from fp32 sums on the GPU and fp64 in the
    # oracle, so a code may differ where the value sits at a rounding tie.
    for name, x in (("q", q), ("k", k)):
        assert np.array_equal(got[name + "_scale"].cpu().numpy(), ref[name + "_scale"]), name
        assert ref[name + "_scale"].shape[2] == (N + 127) // 128
        gc = got[name + "8"].cpu().numpy()
        if rot:
            exact = oracle.hadamard_rotate(x, s)
            sc = np.repeat(ref[name + "_scale"].transpose(0, 2, 1), 128, axis=1)[:, :N, :, None]
            compare_codes(gc, ref[name + "8"], exact / sc, f"{name} codes")
        else:
            assert np.array_equal(gc, ref[name + "8"]), name
    assert np.array_equal(got["v_scale"].cpu().numpy(), ref["v_scale"])
    vt = got["vt8"].cpu().numpy()[..., :N].transpose(0, 3, 1, 2)
    assert np.array_equal(vt, ref["v8"])


CASES = [
    # B, N, Hq, Hkv, causal, window
    (1, 1, 2, 1, 1, 0),
    (1, 129, 2, 2, 0, 0),
    (2, 300, 4, 2, 1, 0),
    (1, 640, 4, 1, 1, 0),
    (1, 513, 4, 2, 0, 0),
    (1, 1000, 2, 2, 1, 200),
    (1, 777, 8, 2, 1, 1),
]


@pytest.mark.parametrize("B,N,Hq,Hkv,causal,window", CASES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_fwd_fp8_on_oracle_codes(fa, B, N, Hq, Hkv, causal, window, out_dtype):
    q, k, v = inputs(B, N, Hq, Hkv, seed=3 * N + Hq)
    p = oracle.fp8_prepare(q, k, v, signs(128, 5))
    scale = 1.0 / math.sqrt(128)
    o, lse = fa.fwd_fp8(to_device_prep(p, N), causal, window, scale, out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.attn_fp8(p["q8"], p["q_scale"], p["k8"], p["k_scale"], p["v8"],
                                     p["v_scale"], causal, window, scale)
    a_ref, _ = oracle.attn_fp8(p["q8"], p["q_scale"], p["k8"], p["k_scale"], abs_v(p),
                               p["v_scale"], causal, window, scale)
    compare_fp8(o, o_ref, a_ref, lse, lse_ref, f"fp8 N={N} causal={causal} W={window}")


@pytest.mark.parametrize("rot", [False, True])
def test_fp8_end_to_end(fa, rot):
    """fa_fp8_prepare then fa_fwd_fp8 against the oracle's whole FP8 prefill.
    Without the rotation the GPU's codes are the oracle's, bit for bit; with
    it a code may differ at a rounding tie (test_prepare_matches_oracle), and
    the tolerance widens by the score shift those codes can cause."""
    B, N, Hq, Hkv = 1, 700, 8, 2
    q, k, v = inputs(B, N, Hq, Hkv, seed=71)
    s = signs(128, 72) if rot else None
    scale = 1.0 / math.sqrt(128)
    o_ref, lse_ref, p = oracle.fp8_prefill(q, k, v, s, causal=True, scale=scale)
    a_ref, _ = oracle.attn_fp8(p["q8"], p["q_scale"], p["k8"], p["k_scale"], abs_v(p),
                               p["v_scale"], True, 0, scale)
    sg = torch.tensor(s, dtype=torch.float32).cuda() if rot else None
    prep = fa.fp8_prepare(q.cuda(), k.cuda(), v.cuda(), sg)
    o, lse = fa.fwd_fp8(prep, True, 0, scale)
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    q8, k8 = prep["q8"].cpu().numpy(), prep["k8"].cpu().numpy()
    if not rot:
        assert np.array_equal(q8, p["q8"]) and np.array_equal(k8, p["k8"])
        compare_fp8(o, o_ref, a_ref, lse, lse_ref, "fp8 end to end")
        return
    assert (q8 != p["q8"]).mean() <= 1e-3 and (k8 != p["k8"]).mean() <= 1e-3
    ds = code_flip_score_bound(q8, p["q8"], p["q_scale"], k8, p["k8"], p["k_scale"], scale,
                               True, 0)
    vmax = float(np.abs(np.array([oracle.e4m3_value(c) for c in range(256)])[p["v8"]]).max()
                 * p["v_scale"].max())
    compare_fp8(o, o_ref, a_ref, lse, lse_ref, "fp8 end to end, rotated", ds=ds, vmax=vmax)


def test_rotation_lowers_gpu_error_with_outliers(fa):
    """The pages' claim on the GPU's own results: with outlier channels in Q
    and K, the rotated FP8 prefill is closer to exact attention than plain FP8."""
    B, N, Hq, Hkv = 1, 512, 4, 2
    q, k, v = inputs(B, N, Hq, Hkv, seed=81, outliers=True)
    scale = 0.1 / math.sqrt(128)
    ref, _ = oracle.attn(q, k, v, True, 0, scale)
    errs = []
    for s in (None, signs(128, 82)):
        sg = torch.tensor(s, dtype=torch.float32).cuda() if s is not None else None
        prep = fa.fp8_prepare(q.cuda(), k.cuda(), v.cuda(), sg)
        o, _ = fa.fwd_fp8(prep, True, 0, scale, out_dtype=torch.float32)
        errs.append(float(np.sqrt(((to64(o) - ref) ** 2).mean())))
    assert errs[1] * 2.0 < errs[0], errs


def test_fp8_gqa4k_full_size(fa):
    """The benchmark's shape (B=1, Hq=32, Hkv=8, N=4096, d=128, causal) in the
    benchmark's launch: fa_fp8_prepare's scales and codes against the
    oracle's in full, fa_fwd_fp8 on the oracle's codes on sampled rows."""
    inp = workloads.make("gqa4k", seed=0)
    s = workloads.hadamard_signs(128, seed=0)
    p = oracle.fp8_prepare(inp.q, inp.k, inp.v, s.numpy().astype(np.float64))
    prep = fa.fp8_prepare(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), s.cuda())
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    N = inp.q.shape[1]
    for name, x in (("q", inp.q), ("k", inp.k)):
        assert np.array_equal(prep[name + "_scale"].cpu().numpy(), p[name + "_scale"]), name
        sc = np.repeat(p[name + "_scale"].transpose(0, 2, 1), 128, axis=1)[:, :N, :, None]
        compare_codes(prep[name + "8"].cpu().numpy(), p[name + "8"],
                      oracle.hadamard_rotate(x, s.numpy().astype(np.float64)) / sc,
                      f"gqa4k {name} codes")
    assert np.array_equal(prep["v_scale"].cpu().numpy(), p["v_scale"])
    assert np.array_equal(prep["vt8"].cpu().numpy()[..., :N].transpose(0, 3, 1, 2), p["v8"])
    o, lse = fa.fwd_fp8(to_device_prep(p, N), True, 0, inp.scale)
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    assert torch.isfinite(o.float()).all()
    rows = [0, 1, 127, 128, 255, 256, 1000, 2047, 2048, 3000, 4094, 4095]
    o_ref, lse_ref = oracle.attn_fp8(p["q8"], p["q_scale"], p["k8"], p["k_scale"], p["v8"],
                                     p["v_scale"], True, 0, inp.scale, rows=rows)
    a_ref, _ = oracle.attn_fp8(p["q8"], p["q_scale"], p["k8"], p["k_scale"], abs_v(p),
                               p["v_scale"], True, 0, inp.scale, rows=rows)
    compare_fp8(o[:, rows], o_ref, a_ref, lse[:, :, rows], lse_ref, "gqa4k fp8 sampled")
