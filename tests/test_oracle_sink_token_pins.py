"""Pins for the oracle's sink tokens: a sliding window of W keys that also
keeps the first n_sink tokens of each sequence visible (samanvya.dev
"Attention Is the Bottleneck", "Sliding windows and local:global layers":
StreamingLLM retains the first few tokens as sinks beside the recent
window).  Pins, none
produced by the oracle itself:
  - torch's softmax in fp64 over the explicitly masked score matrix (a
    library routine for the definition);
  - Q = 0 gives uniform weights over the visible set: LSE_i = log |A(i)| with
    |A(i)| = min(i+1, W) + min(n_sink, max(0, i+1-W)), and O_i the mean of V
    over A(i);
  - n_sink = 0 is the plain window; n_sink >= N, or W >= N, is causal.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def torch_ref(q, k, v, W, S, scale):
    B, N, Hq, d = q.shape
    g = Hq // k.shape[2]
    kk = k.double().repeat_interleave(g, dim=2)
    vv = v.double().repeat_interleave(g, dim=2)
    s = torch.einsum("bihc,bjhc->bhij", q.double(), kk) * scale
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    vis = (j <= i) & ((j > i - W) | (j < S))
    s = s.masked_fill(~vis, float("-inf"))
    o = torch.einsum("bhij,bjhc->bihc", torch.softmax(s, dim=-1), vv)
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


@pytest.mark.parametrize("N,W,S", [(50, 8, 3), (70, 16, 1), (64, 20, 30), (90, 5, 0), (40, 7, 200)])
def test_matches_torch_masked_softmax(N, W, S):
    q, k, v = rnd((2, N, 4, 16), N), rnd((2, N, 2, 16), N + 1), rnd((2, N, 2, 16), N + 2)
    o, lse = oracle.attn_sink_tokens(q, k, v, W, S, 0.3)
    ro, rl = torch_ref(q, k, v, W, S, 0.3)
    assert np.abs(o - ro).max() < 1e-12
    assert np.abs(lse - rl).max() < 1e-12


def test_zero_queries_closed_form():
    N, W, S = 60, 9, 4
    q = torch.zeros((1, N, 2, 8), dtype=torch.bfloat16)
    k, v = rnd((1, N, 1, 8), 5), rnd((1, N, 1, 8), 6)
    o, lse = oracle.attn_sink_tokens(q, k, v, W, S, 1.0)
    vd = v.double().numpy()[0, :, 0]
    for i in range(N):
        vis = [j for j in range(i + 1) if j > i - W or j < S]
        assert len(vis) == min(i + 1, W) + min(S, max(0, i + 1 - W))
        assert abs(lse[0, 0, i] - math.log(len(vis))) < 1e-13
        assert np.abs(o[0, i, 0] - vd[vis].mean(axis=0)).max() < 1e-13


def test_reductions_to_window_and_causal():
    N = 45
    q, k, v = rnd((1, N, 2, 16), 7), rnd((1, N, 2, 16), 8), rnd((1, N, 2, 16), 9)
    a = oracle.attn_sink_tokens(q, k, v, 6, 0, 0.25)
    b = oracle.attn(q, k, v, True, 6, 0.25)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))
    c = oracle.attn(q, k, v, True, 0, 0.25)
    for W, S in ((6, N), (N, 3)):
        d_ = oracle.attn_sink_tokens(q, k, v, W, S, 0.25)
        assert all(np.array_equal(x, y) for x, y in zip(d_, c))


def test_packed_sequences_are_per_sequence():
    """Packed form: each sequence's rows equal the pinned dense form on that
    sequence alone (sink tokens are each sequence's own first tokens)."""
    lens = [70, 0, 130, 5]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    q, k, v = rnd((T, 4, 16), 11), rnd((T, 2, 16), 12), rnd((T, 2, 16), 13)
    o, lse = oracle.attn_varlen_sink_tokens(q, k, v, cu, 9, 3, 0.3)
    for s, L in enumerate(lens):
        if L == 0:
            continue
        a, b = int(cu[s]), int(cu[s + 1])
        ro, rl = oracle.attn_sink_tokens(q[None, a:b], k[None, a:b], v[None, a:b], 9, 3, 0.3)
        assert np.array_equal(o[a:b], ro[0]) and np.array_equal(lse[:, a:b], rl[0])
