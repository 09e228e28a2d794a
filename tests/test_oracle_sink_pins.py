"""Pins for the oracle's learned attention sink: a per-head logit z_h that
joins every row's softmax denominator as the score of one extra key whose
value is zero (samanvya.dev "Attention Is the Bottleneck", "Sliding windows
and local:global layers": gpt-oss builds a learned sink into every head; the
page gives no formula, this is the plain reading).  Pins, none produced by the oracle:
  - z = -inf is plain attention, bit for bit;
  - z equals a real extra key with score z and a zero value, built from the
    plain (pinned) oracle on an augmented input;
  - the closed form with Q = 0: P = 1 / (|A(i)| + e^z), LSE = log(|A(i)| + e^z).
"""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def test_minus_inf_sink_is_plain_attention():
    q, k, v = rnd((2, 50, 4, 32), 1), rnd((2, 50, 2, 32), 2), rnd((2, 50, 2, 32), 3)
    for causal, window in ((0, 0), (1, 0), (1, 7)):
        o, l = oracle.attn(q, k, v, causal, window, 0.2)
        o2, l2 = oracle.attn_sinks(q, k, v, [-math.inf] * 4, causal, window, 0.2)
        assert np.array_equal(o, o2) and np.array_equal(l, l2)


@pytest.mark.parametrize("causal", [0, 1])
def test_sink_equals_extra_zero_value_key(causal):
    """d = 2, scale = 1: q_i = (a_i, 1), real keys (b_j, 0), and one extra key
    (0, z) placed first, with value 0: its score is z for every query.  With
    causal masking the extra token sits at position 0, visible to all."""
    N, z = 24, 0.75
    g = torch.Generator("cpu").manual_seed(7)
    a = torch.randn(N, generator=g)
    b = torch.randn(N, generator=g)
    vals = torch.randn(N, 2, generator=g)
    q = torch.stack([a, torch.ones(N)], -1).to(torch.bfloat16).view(1, N, 1, 2)
    k = torch.stack([b, torch.zeros(N)], -1).to(torch.bfloat16).view(1, N, 1, 2)
    v = vals.to(torch.bfloat16).view(1, N, 1, 2)
    o, lse = oracle.attn_sinks(q, k, v, [z], causal, 0, 1.0)
    # augmented input: token 0 is the sink key; query 0 is a dummy row
    qa = torch.cat([torch.zeros(1, 1, 1, 2, dtype=torch.bfloat16), q], 1)
    ka = torch.cat([torch.tensor([0.0, z]).to(torch.bfloat16).view(1, 1, 1, 2), k], 1)
    va = torch.cat([torch.zeros(1, 1, 1, 2, dtype=torch.bfloat16), v], 1)
    oa, la = oracle.attn(qa, ka, va, causal, 0, 1.0)
    np.testing.assert_allclose(o, oa[:, 1:], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, la[:, :, 1:], rtol=0, atol=1e-14)


def test_sink_closed_form_zero_queries():
    N, Hq, d = 40, 2, 16
    q = torch.zeros(1, N, Hq, d, dtype=torch.bfloat16)
    k, v = rnd((1, N, 1, d), 11), rnd((1, N, 1, d), 12)
    z = [1.5, -2.0]
    o, lse = oracle.attn_sinks(q, k, v, z, 1, 0, 0.3)
    vv = v.double().numpy()[0, :, 0]
    for h in range(Hq):
        for i in range(N):
            den = (i + 1) + math.exp(z[h])
            assert abs(lse[0, h, i] - math.log(den)) < 1e-13
            ref = vv[: i + 1].sum(0) / den
            assert np.abs(o[0, i, h] - ref).max() < 1e-13


def test_decode_sink_matches_last_row_of_prefill():
    """One query at the last position over a paged cache equals the last row
    of the causal prefill with the same sink (identity-mapped pages)."""
    L, Hq, Hkv, d, ps = 37, 4, 2, 32, 16
    q, k, v = rnd((1, L, Hq, d), 21), rnd((1, L, Hkv, d), 22), rnd((1, L, Hkv, d), 23)
    z = [0.3, -0.7, 2.0, -math.inf]
    o, lse = oracle.attn_sinks(q, k, v, z, 1, 0, 0.25)
    npg = -(-L // ps)
    kc = torch.zeros(npg * ps, Hkv, d, dtype=torch.bfloat16)
    vc = torch.zeros(npg * ps, Hkv, d, dtype=torch.bfloat16)
    kc[:L], vc[:L] = k[0], v[0]
    bt = torch.arange(npg, dtype=torch.int32).view(1, npg)
    od, ld = oracle.decode_paged_sinks(q[0, L - 1:L], kc.view(npg, ps, Hkv, d),
                                       vc.view(npg, ps, Hkv, d), bt,
                                       torch.tensor([L], dtype=torch.int32), z, 0.25)
    assert np.abs(od[0] - o[0, L - 1]).max() < 1e-14
    assert np.abs(ld[0] - lse[0, :, L - 1]).max() < 1e-14
