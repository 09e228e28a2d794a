"""Pins for the oracle's attention backward (dQ, dK, dV for an upstream dO).

The pages state only that the backward rebuilds the attention matrix from
the inputs and the forward's row statistics rather than storing it
(samanvya.dev "Attention Is the Bottleneck", "FlashAttention: same math,
different IO"); the gradients
themselves are fixed by calculus.  Pins, none produced by the oracle:
  - hand-worked gradients of the two-key case (tests/golden);
  - torch's automatic differentiation, in fp64, of the forward definition
    (a library routine for the derivative, independent of the oracle's
    analytic formulas), over every mask kind, GQA, both head sizes, varlen;
  - invariants of the exact gradient: the softmax rows sum to one, so
    sum_j dK_j = 0 and sum_j dV_j = sum of dO over the group's query rows;
    a row that sees one key has dS = 0, so it adds nothing to dQ or dK.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed, std=1.0):
    g = torch.Generator("cpu").manual_seed(seed)
    return (torch.randn(shape, generator=g) * std).to(torch.bfloat16)


def autograd_grads(q, k, v, dout, causal, window, scale):
    """fp64 autograd of softmax(QK^T*scale + mask)V for one dense batch."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    qd = q.double().requires_grad_()
    kd = k.double().requires_grad_()
    vd = v.double().requires_grad_()
    kk = kd.repeat_interleave(Hq // Hkv, dim=2)
    vv = vd.repeat_interleave(Hq // Hkv, dim=2)
    s = torch.einsum("bihc,bjhc->bhij", qd, kk) * scale
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    allowed = torch.ones(N, N, dtype=torch.bool)
    if causal:
        allowed &= j <= i
        if window > 0:
            allowed &= j > i - window
    s = s.masked_fill(~allowed, float("-inf"))
    o = torch.einsum("bhij,bjhc->bihc", torch.softmax(s, dim=-1), vv)
    (o * dout.double()).sum().backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy()


def test_backward_hand_cases():
    spec = json.load(open(os.path.join(GOLD, "backward_hand_cases.json")))
    q = torch.tensor(spec["q"]).reshape(1, 2, 1, 1).to(torch.bfloat16)
    k = torch.tensor(spec["k"]).reshape(1, 2, 1, 1).to(torch.bfloat16)
    v = torch.tensor(spec["v"]).reshape(1, 2, 1, 1).to(torch.bfloat16)
    for case in spec["cases"]:
        do = torch.tensor(case["do"]).reshape(1, 2, 1, 1).to(torch.bfloat16)
        dq, dk, dv = oracle.attn_bwd(q, k, v, do, case["causal"], 0, spec["scale"])
        np.testing.assert_allclose(dq.ravel(), case["dq"], atol=1e-14, err_msg=case["name"])
        np.testing.assert_allclose(dk.ravel(), case["dk"], atol=1e-14, err_msg=case["name"])
        np.testing.assert_allclose(dv.ravel(), case["dv"], atol=1e-14, err_msg=case["name"])


@pytest.mark.parametrize("B,N,Hq,Hkv,d,causal,window", [
    (1, 33, 2, 2, 16, 0, 0),
    (2, 40, 4, 1, 8, 1, 0),
    (1, 57, 4, 2, 64, 1, 7),
    (1, 24, 2, 1, 128, 1, 1),
    (1, 30, 8, 2, 32, 1, 64),
])
def test_backward_matches_autograd(B, N, Hq, Hkv, d, causal, window):
    seed = B * 1000 + N * 10 + d
    q, k, v = rnd((B, N, Hq, d), seed), rnd((B, N, Hkv, d), seed + 1), rnd((B, N, Hkv, d), seed + 2)
    do = rnd((B, N, Hq, d), seed + 3)
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal, window, scale)
    rq, rk, rv = autograd_grads(q, k, v, do, causal, window, scale)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_backward_varlen_is_per_sequence():
    """Packed sequences: each sequence's gradients equal a dense run of it alone."""
    lens = [5, 0, 17, 9]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv, d = int(cu[-1]), 4, 2, 16
    q, k, v = rnd((T, Hq, d), 1), rnd((T, Hkv, d), 2), rnd((T, Hkv, d), 3)
    do = rnd((T, Hq, d), 4)
    dq, dk, dv = oracle.attn_bwd_varlen(q, k, v, do, cu, True, 0, 0.25)
    for s, L in enumerate(lens):
        if L == 0:
            continue
        a, b = int(cu[s]), int(cu[s + 1])
        rq, rk, rv = autograd_grads(q[None, a:b], k[None, a:b], v[None, a:b], do[None, a:b],
                                    True, 0, 0.25)
        assert np.abs(dq[a:b] - rq[0]).max() < 1e-12
        assert np.abs(dk[a:b] - rk[0]).max() < 1e-12
        assert np.abs(dv[a:b] - rv[0]).max() < 1e-12


@pytest.mark.parametrize("causal,window", [(0, 0), (1, 0), (1, 5)])
def test_backward_invariants(causal, window):
    B, N, Hq, Hkv, d = 1, 48, 6, 2, 32
    q, k, v = rnd((B, N, Hq, d), 11), rnd((B, N, Hkv, d), 12), rnd((B, N, Hkv, d), 13)
    do = rnd((B, N, Hq, d), 14)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, causal, window, 0.2)
    g = Hq // Hkv
    # sum_j dS_ij = 0 for every row, hence sum_j dK_j = 0 per KV head
    assert np.abs(dk.sum(axis=1)).max() < 1e-12
    # rows of P sum to one, hence sum_j dV_j = sum over the group's dO rows
    dsum = do.double().numpy().reshape(B, N, Hkv, g, d).sum(axis=(1, 3))
    assert np.abs(dv.sum(axis=1) - dsum).max() < 1e-11
    if causal:
        # row 0 sees only key 0: dS = 0, so dQ_0 = 0
        assert np.abs(dq[:, 0]).max() == 0.0


def test_backward_window_one_is_identity_map():
    """W = 1: O_i = V_i, so dV = the group's dO, and dQ = dK = 0."""
    B, N, Hq, Hkv, d = 1, 20, 4, 2, 16
    q, k, v = rnd((B, N, Hq, d), 21), rnd((B, N, Hkv, d), 22), rnd((B, N, Hkv, d), 23)
    do = rnd((B, N, Hq, d), 24)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, 1, 1, 0.3)
    assert np.abs(dq).max() == 0.0 and np.abs(dk).max() == 0.0
    ref = do.double().numpy().reshape(B, N, Hkv, 2, d).sum(axis=3)
    assert np.abs(dv - ref).max() < 1e-14


def test_backward_thread_count_does_not_change_bits():
    B, N, Hq, Hkv, d = 1, 64, 4, 2, 32
    q, k, v = rnd((B, N, Hq, d), 31), rnd((B, N, Hkv, d), 32), rnd((B, N, Hkv, d), 33)
    do = rnd((B, N, Hq, d), 34)
    n0 = oracle.max_threads()
    try:
        oracle.set_num_threads(1)
        a = oracle.attn_bwd(q, k, v, do, 1, 0, 0.125)
        oracle.set_num_threads(max(2, n0))
        b = oracle.attn_bwd(q, k, v, do, 1, 0, 0.125)
    finally:
        oracle.set_num_threads(n0)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_dq_rows_match_full_backward():
    """The row-sampled dQ equals the pinned full backward on the same rows."""
    lens = [40, 0, 77]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv, d = int(cu[-1]), 4, 2, 32
    q, k, v = rnd((T, Hq, d), 41), rnd((T, Hkv, d), 42), rnd((T, Hkv, d), 43)
    do = rnd((T, Hq, d), 44)
    for causal, window in ((0, 0), (1, 0), (1, 9)):
        dq, _, _ = oracle.attn_bwd_varlen(q, k, v, do, cu, causal, window, 0.3)
        rows = [0, 5, 39, 40, 41, 100, 116]
        got = oracle.attn_bwd_dq_rows(q, k, v, do, cu, rows, causal, window, 0.3)
        assert np.array_equal(got, dq[rows])


def autograd_grads_sinks(q, k, v, dout, sinks, causal, window, scale):
    """fp64 autograd with the sink as one extra score column (value zero)."""
    B, N, Hq, d = q.shape
    Hkv = k.shape[2]
    qd = q.double().requires_grad_()
    kd = k.double().requires_grad_()
    vd = v.double().requires_grad_()
    z = torch.tensor(sinks, dtype=torch.float64).requires_grad_()
    kk = kd.repeat_interleave(Hq // Hkv, dim=2)
    vv = vd.repeat_interleave(Hq // Hkv, dim=2)
    s = torch.einsum("bihc,bjhc->bhij", qd, kk) * scale
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    allowed = torch.ones(N, N, dtype=torch.bool)
    if causal:
        allowed &= j <= i
        if window > 0:
            allowed &= j > i - window
    s = s.masked_fill(~allowed, float("-inf"))
    zc = z.view(1, Hq, 1, 1).expand(B, Hq, N, 1)
    pr = torch.softmax(torch.cat([s, zc], dim=-1), dim=-1)[..., :N]
    o = torch.einsum("bhij,bjhc->bihc", pr, vv)
    (o * dout.double()).sum().backward()
    return qd.grad.numpy(), kd.grad.numpy(), vd.grad.numpy(), z.grad.numpy()


@pytest.mark.parametrize("causal,window", [(0, 0), (1, 0), (1, 6)])
def test_backward_with_sinks_matches_autograd(causal, window):
    B, N, Hq, Hkv, d = 2, 29, 4, 2, 16
    q, k, v = rnd((B, N, Hq, d), 51), rnd((B, N, Hkv, d), 52), rnd((B, N, Hkv, d), 53)
    do = rnd((B, N, Hq, d), 54)
    z = [0.7, -1.3, 2.5, 0.0]
    dq, dk, dv, dz = oracle.attn_bwd_sinks(q, k, v, do, z, causal, window, 0.25)
    rq, rk, rv, rz = autograd_grads_sinks(q, k, v, do, z, causal, window, 0.25)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv), (dz, rz)):
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_minus_inf_sinks_backward_is_plain():
    B, N, Hq, Hkv, d = 1, 33, 2, 1, 16
    q, k, v = rnd((B, N, Hq, d), 61), rnd((B, N, Hkv, d), 62), rnd((B, N, Hkv, d), 63)
    do = rnd((B, N, Hq, d), 64)
    a = oracle.attn_bwd(q, k, v, do, 1, 0, 0.3)
    b = oracle.attn_bwd_sinks(q, k, v, do, [-math.inf, -math.inf], 1, 0, 0.3)
    for x, y in zip(a, b[:3]):
        assert np.array_equal(x, y)
    assert np.all(b[3] == 0.0)



def test_dkv_rows_match_full_backward():
    """The key-row dK, dV (row statistics first, then per-key sums over the
    rows that see the key) equal the pinned full backward's rows, which
    scatters each query row's terms into every key it sees."""
    lens = [40, 0, 77]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T, Hq, Hkv, d = int(cu[-1]), 4, 2, 32
    q, k, v = rnd((T, Hq, d), 51), rnd((T, Hkv, d), 52), rnd((T, Hkv, d), 53)
    do = rnd((T, Hq, d), 54)
    rows = [0, 5, 39, 40, 41, 100, 116]
    for causal, window in ((0, 0), (1, 0), (1, 9), (1, 1)):
        _, dk, dv = oracle.attn_bwd_varlen(q, k, v, do, cu, causal, window, 0.3)
        gk, gv = oracle.attn_bwd_dkv_rows(q, k, v, do, cu, rows, causal, window, 0.3)
        for got, ref in ((gk, dk[rows]), (gv, dv[rows])):
            assert np.allclose(got, ref, rtol=1e-12, atol=1e-13 * np.abs(ref).max())
    # a window of one key: each key is seen only by its own row, whose softmax
    # is that key alone, so dS = 0 (dK = 0) and dV_j sums dO_j over the
    # group's query heads
    gk, gv = oracle.attn_bwd_dkv_rows(q, k, v, do, cu, rows, 1, 1, 0.3)
    assert np.abs(gk).max() == 0.0
    dod = do.double().numpy().reshape(T, Hkv, Hq // Hkv, d).sum(axis=2)
    assert np.allclose(gv, dod[rows], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window", [(0, 0), (1, 0), (1, 5)])
def test_dkv_rows_match_autograd(causal, window):
    """Independent of the oracle's other backward: fp64 autograd of the
    forward definition, on a dense GQA batch, at chosen key rows."""
    B, N, Hq, Hkv, d = 1, 33, 4, 2, 16
    q, k, v = rnd((B, N, Hq, d), 61), rnd((B, N, Hkv, d), 62), rnd((B, N, Hkv, d), 63)
    do = rnd((B, N, Hq, d), 64)
    _, dk_ref, dv_ref = autograd_grads(q, k, v, do, causal, window, 0.25)
    rows = [0, 1, 16, 31, 32]
    cu = np.array([0, N], dtype=np.int32)
    gk, gv = oracle.attn_bwd_dkv_rows(q[0], k[0], v[0], do[0], cu, rows, causal, window, 0.25)
    assert np.allclose(gk, dk_ref[0, rows], rtol=1e-10, atol=1e-12)
    assert np.allclose(gv, dv_ref[0, rows], rtol=1e-10, atol=1e-12)
