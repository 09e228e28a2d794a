"""GPU parity of the attention backward (fa_bwd / fa_bwd_varlen) against the
fp64 oracle's gradients, on the same seeded inputs, through the C ABI.

The forward's own outputs (O and LSE from fa_fwd) feed the backward, as in
training.  Tolerance, per gradient tensor G (derived from the arithmetic:
P and dS enter the tensor-core GEMMs as bf16, relative rounding 2^-9 per
term, O enters D_i = dO_i . O_i as bf16, and the results are rounded to
bf16, 2^-9 relative):
    max |G_gpu - G_ref| <= 2e-2 * max |G_ref| + 1e-4
    mean |G_gpu - G_ref| <= 1e-2 * mean |G_ref| + 1e-5
The absolute floors cover gradients that are exactly zero (a window of one
key makes dS = 0): there dP_ij - D_i is a difference of two fp32 sums of the
same 128 products taken in different orders, ~1e-6 of |dO||V|.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu

TOL_MAX_REL = 2e-2
TOL_MEAN_REL = 1e-2
TOL_MAX_ABS = 1e-4
TOL_MEAN_ABS = 1e-5


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_io_aware_75_b200 as fa
    return fa


def check(name, got, ref, what):
    g = got.detach().float().cpu().double().numpy()
    assert g.shape == ref.shape, (what, name, g.shape, ref.shape)
    assert np.all(np.isfinite(g)), f"{what} {name}: non-finite"
    err = np.abs(g - ref)
    mx_ref, mean_ref = np.abs(ref).max(), np.abs(ref).mean()
    assert err.max() <= TOL_MAX_REL * mx_ref + TOL_MAX_ABS, \
        f"{what} {name}: max err {err.max():.3e} vs max|ref| {mx_ref:.3e}"
    assert err.mean() <= TOL_MEAN_REL * mean_ref + TOL_MEAN_ABS, \
        f"{what} {name}: mean err {err.mean():.3e} vs mean|ref| {mean_ref:.3e}"
    return float(err.max() / max(mx_ref, 1e-30)), float(err.mean() / max(mean_ref, 1e-30))


def run_dense(fa, inp, do):
    q, k, v, dO = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), do.cuda()
    o, lse = fa.fwd(q, k, v, inp.causal, inp.window, inp.scale)
    dq, dk, dv = fa.bwd(q, k, v, o, dO, lse, inp.causal, inp.window, inp.scale)
    assert fa.check_device_error() == 0
    return dq, dk, dv


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,window", [
    (1, 2, 2, 64, True, 0),
    (1, 2, 2, 128, False, 0),
    (1, 4, 2, 300, True, 0),
    (1, 2, 1, 200, False, 0),
    (2, 8, 2, 257, True, 0),
    (1, 4, 1, 700, True, 130),
    (1, 2, 2, 513, True, 1),
    (1, 4, 4, 1024, True, 0),
    (1, 2, 2, 1, True, 0),
])
def test_dense(fa, B, Hq, Hkv, N, causal, window):
    inp = workloads.dense(B, Hq, Hkv, N, 128, causal=causal, window=window, seed=N + Hq)
    do = workloads.grad_out((B, N, Hq, 128), seed=N + Hq)
    dq, dk, dv = run_dense(fa, inp, do)
    rq, rk, rv = oracle.attn_bwd(inp.q, inp.k, inp.v, do, causal, window, inp.scale)
    what = f"B={B} Hq={Hq} Hkv={Hkv} N={N} causal={causal} W={window}"
    check("dQ", dq, rq, what)
    check("dK", dk, rk, what)
    check("dV", dv, rv, what)


def test_varlen(fa):
    lens = [100, 0, 333, 64, 1, 200]
    inp = workloads.varlen(lens=lens, Hq=4, Hkv=2, d=128, causal=True, seed=5)
    T = sum(lens)
    do = workloads.grad_out((T, 4, 128), seed=5)
    q, k, v, dO = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), do.cuda()
    cu = inp.cu_seqlens.cuda()
    o, lse = fa.fwd_varlen(q, k, v, cu, inp.max_seqlen, True, 0, inp.scale)
    dq, dk, dv = fa.bwd_varlen(q, k, v, o, dO, lse, cu, inp.max_seqlen, True, 0, inp.scale)
    assert fa.check_device_error() == 0
    rq, rk, rv = oracle.attn_bwd_varlen(inp.q, inp.k, inp.v, do, inp.cu_seqlens, True, 0,
                                        inp.scale)
    check("dQ", dq, rq, "varlen")
    check("dK", dk, rk, "varlen")
    check("dV", dv, rv, "varlen")


def test_gqa_equals_repeated_heads(fa):
    """GQA gradients: dK, dV of a KV head equal the sum over its query heads
    of an MHA run with K, V repeated; dQ is the same."""
    B, Hq, Hkv, N = 1, 8, 2, 384
    inp = workloads.dense(B, Hq, Hkv, N, 128, causal=True, seed=21)
    do = workloads.grad_out((B, N, Hq, 128), seed=21).cuda()
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    o, lse = fa.fwd(q, k, v, True, 0, inp.scale)
    dq, dk, dv = fa.bwd(q, k, v, o, do, lse, True, 0, inp.scale)
    kr, vr = k.repeat_interleave(4, dim=2).contiguous(), v.repeat_interleave(4, dim=2).contiguous()
    o2, lse2 = fa.fwd(q, kr, vr, True, 0, inp.scale)
    dq2, dk2, dv2 = fa.bwd(q, kr, vr, o2, do, lse2, True, 0, inp.scale)
    assert fa.check_device_error() == 0
    sk = dk2.float().view(B, N, Hkv, 4, 128).sum(3)
    sv = dv2.float().view(B, N, Hkv, 4, 128).sum(3)
    assert (dk.float() - sk).abs().max().item() <= 2e-2 * sk.abs().max().item()
    assert (dv.float() - sv).abs().max().item() <= 2e-2 * sv.abs().max().item()
    assert (dq.float() - dq2.float()).abs().max().item() <= 1e-2 * dq2.float().abs().max().item()


def test_dk_dv_deterministic(fa):
    inp = workloads.dense(1, 4, 2, 640, 128, causal=True, seed=3)
    do = workloads.grad_out((1, 640, 4, 128), seed=3)
    a = run_dense(fa, inp, do)
    b = run_dense(fa, inp, do)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_gqa4k_full_size(fa):
    """The full 4k GQA shape (B=1, Hq=32, Hkv=8, N=4096, d=128, causal, seed 0):
    sampled dQ rows (every query head) and sampled dK, dV key rows (every KV
    head) element by element against the oracle's row gradients, plus the
    properties the exact gradient has at any size, per KV head:
    sum_j dK_j = 0, and sum_j dV_j = the group's dO summed over all rows."""
    inp = workloads.make("gqa4k", seed=0)
    B, N, Hq, d = inp.q.shape
    Hkv = inp.k.shape[2]
    do = workloads.grad_out((B, N, Hq, d), seed=0)
    dq, dk, dv = run_dense(fa, inp, do)
    g = torch.Generator("cpu").manual_seed(1)
    rows = sorted(set([0, 1, 63, 64, 127, 128, 2047, 4095] +
                      torch.randint(0, N, (24,), generator=g).tolist()))
    cu = torch.tensor([0, N], dtype=torch.int32)
    rq = oracle.attn_bwd_dq_rows(inp.q[0], inp.k[0], inp.v[0], do[0], cu, rows, True, 0,
                                 inp.scale)
    check("dQ rows", dq[0, rows], rq, "gqa4k")
    g = torch.Generator("cpu").manual_seed(2)
    krows = sorted(set([0, 1, 127, 128, 129, 2048, 4094, 4095] +
                       torch.randint(0, N, (24,), generator=g).tolist()))
    rk, rv = oracle.attn_bwd_dkv_rows(inp.q[0], inp.k[0], inp.v[0], do[0], cu, krows, True, 0,
                                      inp.scale)
    check("dK rows", dk[0, krows], rk, "gqa4k")
    check("dV rows", dv[0, krows], rv, "gqa4k")
    dk64 = dk.double().cpu()[0]                        # [N, Hkv, d]
    assert (dk64.sum(0).abs() <= 1e-3 * dk64.abs().sum(0) + 1e-3).all()
    dv64 = dv.double().cpu()[0]
    ref_v = do.double()[0].view(N, Hkv, Hq // Hkv, d).sum(dim=(0, 2))
    assert ((dv64.sum(0) - ref_v).abs() <= 1e-3 * dv64.abs().sum(0) + 1e-2).all()


def test_sinks_backward(fa):
    """Backward of a forward with learned sinks: dQ, dK, dV and the sink-logit
    gradient against the oracle (dsinks within the same relative bound)."""
    import math
    B, Hq, Hkv, N = 1, 8, 2, 333
    inp = workloads.dense(B, Hq, Hkv, N, 128, causal=True, seed=41)
    do = workloads.grad_out((B, N, Hq, 128), seed=41)
    g = torch.Generator("cpu").manual_seed(41)
    z = torch.randn(Hq, generator=g) * 2.0
    z[0] = -math.inf
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    o, lse = fa.fwd(q, k, v, True, 0, inp.scale, sinks=z.cuda())
    dq, dk, dv, dz = fa.bwd(q, k, v, o, do.cuda(), lse, True, 0, inp.scale, sinks=z.cuda())
    assert fa.check_device_error() == 0
    rq, rk, rv, rz = oracle.attn_bwd_sinks(inp.q, inp.k, inp.v, do, z.double().numpy(), True,
                                           0, inp.scale)
    check("dQ", dq, rq, "sinks")
    check("dK", dk, rk, "sinks")
    check("dV", dv, rv, "sinks")
    got = dz.double().cpu().numpy()
    assert got[0] == 0.0
    assert np.abs(got - rz).max() <= TOL_MAX_REL * np.abs(rz).max() + TOL_MAX_ABS


@pytest.mark.parametrize("B,Hq,Hkv,N,causal,window", [
    (1, 4, 2, 300, True, 0), (2, 2, 2, 257, False, 0), (1, 4, 1, 700, True, 130)])
def test_head_dim_64(fa, B, Hq, Hkv, N, causal, window):
    """d = 64: computed on zero-padded 128-wide tiles."""
    inp = workloads.dense(B, Hq, Hkv, N, 64, causal=causal, window=window, seed=N + 64)
    do = workloads.grad_out((B, N, Hq, 64), seed=N + 64)
    dq, dk, dv = run_dense(fa, inp, do)
    rq, rk, rv = oracle.attn_bwd(inp.q, inp.k, inp.v, do, causal, window, inp.scale)
    what = f"d=64 B={B} Hq={Hq} Hkv={Hkv} N={N} causal={causal} W={window}"
    check("dQ", dq, rq, what)
    check("dK", dk, rk, what)
    check("dV", dv, rv, what)
