"""GPU parity of fa_fwd_sink_tokens (a causal sliding window that keeps the
first n_sink tokens of every sequence visible) against the fp64 oracle,
through the C ABI, with the bf16 tolerances of tests/parity.py."""
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


CASES = [
    # B, N, Hq, Hkv, d, window, n_sink
    (1, 300, 4, 2, 128, 64, 4),
    (2, 513, 4, 1, 128, 128, 1),
    (1, 700, 8, 2, 128, 200, 130),      # sinks span two key blocks
    (1, 1000, 2, 2, 64, 100, 256),
    (1, 257, 2, 1, 128, 32, 300),       # more sinks than tokens: causal
    (1, 1, 2, 1, 128, 8, 4),
    (1, 640, 4, 4, 64, 1, 10),          # a window of one key plus the sinks
    (1, 900, 4, 2, 128, 300, 128),      # sinks exactly one block
]


@pytest.mark.parametrize("B,N,Hq,Hkv,d,W,S", CASES)
def test_sink_tokens_match_oracle(fa, B, N, Hq, Hkv, d, W, S):
    inp = workloads.dense(B, Hq, Hkv, N, d, causal=True, seed=N + W + S)
    o, lse = fa.fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), True, W, inp.scale,
                    out_dtype=torch.float32, sink_tokens=S)
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.attn_sink_tokens(inp.q, inp.k, inp.v, W, S, inp.scale)
    compare(o, o_ref, lse, lse_ref, f"sink tokens N={N} W={W} S={S}")


def test_zero_sinks_is_the_window(fa):
    inp = workloads.dense(1, 4, 2, 700, 128, causal=True, seed=3)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    a = fa.fwd(q, k, v, True, 100, inp.scale, sink_tokens=0)
    b = fa.fwd(q, k, v, True, 100, inp.scale)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_sink_tokens_long32k_sampled_rows(fa):
    """The long-context shape (B=1, Hq=32, Hkv=8, N=32768, d=128) with the
    4,096-token window and four sink tokens: sampled rows, all heads."""
    inp = workloads.make("long32k_w4096", seed=0)
    o, lse = fa.fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), True, inp.window, inp.scale,
                    sink_tokens=4)
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    rows = [0, 3, 4, 4095, 4096, 4099, 4100, 20000, 32767]
    o_ref, lse_ref = oracle.attn_sink_tokens(inp.q, inp.k, inp.v, inp.window, 4, inp.scale,
                                             rows=[(0, r) for r in rows])
    compare(o[0, rows], o_ref, lse[0][:, rows].T, lse_ref, "long32k_w4096 + 4 sink tokens")


@pytest.mark.parametrize("W,S", [(64, 4), (200, 130)])
def test_packed_sequences_match_oracle(fa, W, S):
    """fa_fwd_varlen_sink_tokens: each sequence keeps its own first tokens."""
    inp = workloads.varlen(lens=[300, 0, 517, 1, 129, 1000], Hq=8, Hkv=2, d=128, causal=True,
                           seed=W + S)
    cu = inp.cu_seqlens.cuda()
    o, lse = fa.fwd_varlen(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), cu, inp.max_seqlen, True,
                           W, inp.scale, out_dtype=torch.float32, sink_tokens=S)
    torch.cuda.synchronize()
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_sink_tokens(inp.q, inp.k, inp.v, inp.cu_seqlens, W, S,
                                                    inp.scale)
    compare(o, o_ref, lse, lse_ref, f"packed sink tokens W={W} S={S}")
