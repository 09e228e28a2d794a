"""GPU parity of the prefill kernel (fa_fwd / fa_fwd_varlen) against the
fp64 oracle on the same seeded inputs, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import compare

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_io_aware_75_b200 as fa
    return fa


def run_dense(fa, inp, out_dtype=torch.bfloat16):
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    o, lse = fa.fwd(q, k, v, inp.causal, inp.window, inp.scale, out_dtype=out_dtype)
    assert fa.check_device_error() == 0
    return o, lse


def test_tiny_config(fa):
    """B=1, H=2, N=128, d=64, non-causal, scale 1/8, fp32 O + LSE, seed 0."""
    inp = workloads.make("tiny", seed=0)
    o, lse = run_dense(fa, inp, torch.float32)
    o_ref, lse_ref = oracle.attn(inp.q, inp.k, inp.v, inp.causal, inp.window, inp.scale)
    compare(o, o_ref, lse, lse_ref, "tiny")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 256, 257, 383, 513])
def test_dense_sizes(fa, N, causal, d):
    inp = workloads.dense(1, 2, 2, N, d, causal=causal, seed=N + d)
    o, lse = run_dense(fa, inp)
    o_ref, lse_ref = oracle.attn(inp.q, inp.k, inp.v, causal, 0, inp.scale)
    compare(o, o_ref, lse, lse_ref, f"N={N} causal={causal} d={d}")


@pytest.mark.parametrize("B,Hq,Hkv,N,d,causal", [
    (2, 8, 2, 300, 128, True), (3, 4, 1, 200, 64, False), (1, 6, 3, 640, 128, True),
    (2, 4, 4, 1024, 64, True)])
def test_dense_gqa_batches(fa, B, Hq, Hkv, N, d, causal):
    inp = workloads.dense(B, Hq, Hkv, N, d, causal=causal, seed=7)
    o, lse = run_dense(fa, inp)
    o_ref, lse_ref = oracle.attn(inp.q, inp.k, inp.v, causal, 0, inp.scale)
    compare(o, o_ref, lse, lse_ref, f"B={B} Hq={Hq} Hkv={Hkv} N={N}")


@pytest.mark.parametrize("W", [1, 37, 128, 129, 200, 1000])
def test_window(fa, W):
    inp = workloads.dense(1, 4, 2, 700, 128, causal=True, window=W, seed=W)
    o, lse = run_dense(fa, inp)
    o_ref, lse_ref = oracle.attn(inp.q, inp.k, inp.v, True, W, inp.scale)
    compare(o, o_ref, lse, lse_ref, f"W={W}")


def test_fp32_output_matches_bf16_output(fa):
    inp = workloads.dense(1, 2, 2, 333, 128, causal=True, seed=3)
    o32, l32 = run_dense(fa, inp, torch.float32)
    o16, l16 = run_dense(fa, inp, torch.bfloat16)
    assert torch.equal(l32, l16)
    assert torch.equal(o32.to(torch.bfloat16), o16)


def test_identities(fa):
    """window >= N equals causal; GQA equals MHA with repeated K/V; two runs
    are bitwise identical."""
    inp = workloads.dense(1, 8, 2, 450, 128, causal=True, seed=11)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    oc, lc = fa.fwd(q, k, v, True, 0, inp.scale)
    ow, lw = fa.fwd(q, k, v, True, 450, inp.scale)
    assert torch.equal(oc, ow) and torch.equal(lc, lw)
    ow2, lw2 = fa.fwd(q, k, v, True, 10 ** 6, inp.scale)
    assert torch.equal(oc, ow2) and torch.equal(lc, lw2)
    om, lm = fa.fwd(q, k.repeat_interleave(4, dim=2).contiguous(),
                    v.repeat_interleave(4, dim=2).contiguous(), True, 0, inp.scale)
    assert torch.equal(oc, om) and torch.equal(lc, lm)
    oc2, lc2 = fa.fwd(q, k, v, True, 0, inp.scale)
    assert torch.equal(oc, oc2) and torch.equal(lc, lc2)
    assert fa.check_device_error() == 0


@pytest.mark.parametrize("d,causal,window", [(128, True, 0), (64, True, 0), (128, False, 0),
                                             (128, True, 100)])
def test_varlen(fa, d, causal, window):
    lens = [1, 17, 128, 129, 0, 300, 511, 256]
    inp = workloads.varlen(lens=lens, Hq=4, Hkv=2, d=d, causal=causal, window=window, seed=5)
    q, k, v, cu = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.cu_seqlens.cuda()
    o, lse = fa.fwd_varlen(q, k, v, cu, inp.max_seqlen, causal, window, inp.scale)
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen(inp.q, inp.k, inp.v, inp.cu_seqlens, causal, window,
                                        inp.scale)
    compare(o, o_ref, lse, lse_ref, f"varlen d={d} causal={causal} W={window}")
    # each packed sequence equals its own dense call, bit for bit
    c = inp.cu_seqlens.tolist()
    for s, L in enumerate(lens):
        if L == 0:
            continue
        od, ld = fa.fwd(q[c[s]:c[s + 1]][None].contiguous(), k[c[s]:c[s + 1]][None].contiguous(),
                        v[c[s]:c[s + 1]][None].contiguous(), causal, window, inp.scale)
        assert torch.equal(od[0], o[c[s]:c[s + 1]]), s
        assert torch.equal(ld[0], lse[:, c[s]:c[s + 1]]), s


def test_output_guards_untouched(fa):
    """Outputs written into the middle of larger buffers leave the guard
    regions around them unchanged (no stray stores)."""
    inp = workloads.varlen(lens=[5, 200, 130], Hq=4, Hkv=2, d=128, causal=True, seed=9)
    T = sum(inp.lens)
    g = 4096
    obuf = torch.full((g + T * 4 * 128 + g,), 7.0, dtype=torch.bfloat16, device="cuda")
    lbuf = torch.full((g + 4 * T + g,), 7.0, dtype=torch.float32, device="cuda")
    o = obuf[g:g + T * 4 * 128].view(T, 4, 128)
    lse = lbuf[g:g + 4 * T].view(4, T)
    fa.fwd_varlen(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.cu_seqlens.cuda(), 200, True,
                  0, inp.scale, out=o, lse=lse)
    assert fa.check_device_error() == 0
    assert torch.all(obuf[:g] == 7) and torch.all(obuf[-g:] == 7)
    assert torch.all(lbuf[:g] == 7) and torch.all(lbuf[-g:] == 7)
    o_ref, lse_ref = oracle.attn_varlen(inp.q, inp.k, inp.v, inp.cu_seqlens, True, 0, inp.scale)
    compare(o, o_ref, lse, lse_ref, "guarded")


def sampled_rows(N, W, n_random, seed):
    fixed = {0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 1}
    if W:
        fixed |= {W - 1, W, W + 1}
    g = torch.Generator().manual_seed(seed)
    rnd = set(torch.randint(0, N, (n_random,), generator=g).tolist())
    return sorted(r for r in fixed | rnd if 0 <= r < N)


@pytest.mark.parametrize("name,n_random", [("gqa4k", 120), ("long32k", 40),
                                           ("long32k_w4096", 40)])
def test_full_size_dense_sampled(fa, name, n_random):
    """Full-size workloads in the bench's launch configuration, checked on
    sampled rows (all heads) that the oracle computes one by one."""
    inp = workloads.make(name, seed=0)
    o, lse = run_dense(fa, inp)
    N = inp.q.shape[1]
    rows = sampled_rows(N, inp.window, n_random, seed=1)
    o_ref, lse_ref = oracle.attn_rows(inp.q, inp.k, inp.v, [(0, r) for r in rows],
                                      inp.causal, inp.window, inp.scale)
    o_s = o[0, rows]                        # [R, Hq, d]
    l_s = lse[0][:, rows].T                 # [R, Hq]
    compare(o_s, o_ref, l_s, lse_ref, name)


def test_gqa4k_every_row(fa):
    """The headline workload (B=1, Hq=32, Hkv=8, N=4096, d=128, causal, seed 0)
    in the bench's launch configuration: every row and head of O and LSE
    against the fp64 oracle (the whole score matrix, about 4 s on 16 cores)."""
    inp = workloads.make("gqa4k", seed=0)
    o, lse = run_dense(fa, inp)
    o_ref, lse_ref = oracle.attn(inp.q, inp.k, inp.v, True, 0, inp.scale)
    compare(o, o_ref, lse, lse_ref, "gqa4k every row")


def test_full_size_varlen_sampled(fa):
    inp = workloads.make("varlen16", seed=0)
    q, k, v, cu = inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.cu_seqlens.cuda()
    o, lse = fa.fwd_varlen(q, k, v, cu, inp.max_seqlen, True, 0, inp.scale)
    assert fa.check_device_error() == 0
    c = inp.cu_seqlens.tolist()
    rows = []
    for s in range(len(inp.lens)):
        L = inp.lens[s]
        rows += [c[s] + r for r in {0, 1, 127, 128, L // 2, L - 1}]
    g = torch.Generator().manual_seed(2)
    rows += torch.randint(0, c[-1], (64,), generator=g).tolist()
    rows = sorted(set(rows))
    o_ref, lse_ref = oracle.attn_varlen(inp.q, inp.k, inp.v, inp.cu_seqlens, True, 0,
                                        inp.scale, rows=rows)
    compare(o[rows], o_ref, lse[:, rows].T, lse_ref, "varlen16")
