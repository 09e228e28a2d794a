"""Pins for the fp64 oracle: values and properties fixed by the pages and by
mathematics, none of them produced by the oracle itself.

Sources: samanvya.dev "Attention Is the Bottleneck" -- "What attention costs"
(the definition), "FlashAttention: same math, different IO" (online softmax
worked example and its printed 1.39e-16), "Flash-Decoding" (log-sum-exp merge
of split partials), "MQA and GQA" (grouped heads), "Sliding windows and
local:global layers" (last-W-tokens window), "Paging and prefix sharing"
(paged cache).
"""
import json
import math
import os
from decimal import Decimal, getcontext

import numpy as np
import pytest
import torch

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def bf(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def rnd(shape, seed, lo=None, hi=None):
    g = torch.Generator("cpu").manual_seed(seed)
    if lo is not None:
        return torch.randint(lo, hi + 1, shape, generator=g).to(torch.bfloat16)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def f64(t):
    return t.to(torch.float64).numpy()


def visible(i, j, causal, window):
    if not causal:
        return True
    if j > i:
        return False
    return not (window > 0 and j <= i - window)


# --------------------------------------------------------------- golden hand cases
def test_hand_cases():
    spec = json.load(open(os.path.join(GOLD, "hand_cases.json")))
    assert "What attention costs" in spec["source"]
    for case in spec["cases"]:
        q, k, v = (bf(case[n])[None] for n in ("q", "k", "v"))
        o, lse = oracle.attn(q, k, v, causal=case["causal"], window=case["window"],
                             scale=case["scale"])
        np.testing.assert_allclose(o[0], np.array(case["o"]), rtol=0, atol=1e-12,
                                   err_msg=case["name"])
        np.testing.assert_allclose(lse[0], np.array(case["lse"]), rtol=0, atol=1e-12,
                                   err_msg=case["name"])


# ------------------------------------------------- brute force in 40-digit decimal
def _decimal_attention(q, k, v, causal, window, scale):
    """Independent high-precision path: Decimal exp/ln, per-row sums."""
    getcontext().prec = 40
    N, Hq, d = q.shape
    Hkv = k.shape[1]
    g = Hq // Hkv
    qd, kd, vd = (f64(t) for t in (q, k, v))
    o = np.zeros((N, Hq, d))
    lse = np.zeros((Hq, N))
    sc = Decimal(scale)
    for h in range(Hq):
        for i in range(N):
            keys = [j for j in range(N) if visible(i, j, causal, window)]
            s = []
            for j in keys:
                acc = Decimal(0)
                for c in range(d):
                    acc += Decimal(qd[i, h, c]) * Decimal(kd[j, h // g, c])
                s.append(sc * acc)
            e = [x.exp() for x in s]
            tot = sum(e, Decimal(0))
            for c in range(d):
                o[i, h, c] = float(sum((e[n] * Decimal(vd[j, h // g, c])
                                        for n, j in enumerate(keys)), Decimal(0)) / tot)
            lse[h, i] = float(tot.ln())
    return o, lse


@pytest.mark.parametrize("N,d,Hq,Hkv,causal,window", [
    (1, 3, 1, 1, False, 0), (5, 4, 2, 1, False, 0), (6, 3, 2, 2, True, 0),
    (7, 2, 4, 2, True, 3), (8, 4, 3, 1, True, 1)])
def test_brute_force_decimal(N, d, Hq, Hkv, causal, window):
    q, k, v = rnd((N, Hq, d), 1), rnd((N, Hkv, d), 2), rnd((N, Hkv, d), 3)
    scale = 0.7
    o_ref, lse_ref = _decimal_attention(q, k, v, causal, window, scale)
    o, lse = oracle.attn(q[None], k[None], v[None], causal, window, scale)
    np.testing.assert_allclose(o[0], o_ref, rtol=0, atol=2e-14)
    np.testing.assert_allclose(lse[0], lse_ref, rtol=0, atol=2e-14)


# ------------------------------------------------------------------- invariants
@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 5)])
def test_rows_sum_to_one_and_mask(causal, window):
    N, H, d = 23, 2, 16
    q, k, v = rnd((N, H, d), 4), rnd((N, H, d), 5), rnd((N, H, d), 6)
    cu = np.array([0, N], np.int32)
    for h in range(H):
        p = oracle.probs(q, k, v, cu, 0, h, causal, window, 0.25)
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
        for i in range(N):
            for j in range(N):
                if not visible(i, j, causal, window):
                    assert p[i, j] == 0.0
                else:
                    assert p[i, j] > 0.0


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 3)])
def test_constant_v_returns_v(causal, window):
    N, H, d = 19, 2, 8
    q, k = rnd((1, N, H, d), 7), rnd((1, N, H, d), 8)
    v = bf(np.full((1, N, H, d), 0.75))
    o, _ = oracle.attn(q, k, v, causal, window, 0.3)
    np.testing.assert_allclose(o, 0.75, rtol=0, atol=1e-14)


def test_single_key_returns_its_value():
    d = 32
    q, k, v = rnd((1, 1, 2, d), 9), rnd((1, 1, 1, d), 10), rnd((1, 1, 1, d), 11)
    o, lse = oracle.attn(q, k, v, False, 0, 0.125)
    for h in range(2):
        np.testing.assert_array_equal(o[0, 0, h], f64(v)[0, 0, 0])
        dot = math.fsum(float(a) * float(b) for a, b in zip(f64(q)[0, 0, h], f64(k)[0, 0, 0]))
        assert abs(lse[0, h, 0] - 0.125 * dot) < 1e-13


def test_causal_row0_is_v0():
    N, d = 17, 16
    q, k, v = rnd((1, N, 2, d), 12), rnd((1, N, 2, d), 13), rnd((1, N, 2, d), 14)
    o, lse = oracle.attn(q, k, v, True, 0, 0.5)
    np.testing.assert_array_equal(o[0, 0], f64(v)[0, 0])
    for h in range(2):
        dot = math.fsum(float(a) * float(b) for a, b in zip(f64(q)[0, 0, h], f64(k)[0, 0, h]))
        assert abs(lse[0, h, 0] - 0.5 * dot) < 1e-13


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 0), (True, 4)])
def test_zero_query_closed_form(causal, window):
    """Q = 0: all scores 0, so O_i is the plain mean of the visible V rows and
    LSE_i = log |A(i)| (log(i+1), log(min(i+1, W)), log N)."""
    N, d = 21, 8
    q = bf(np.zeros((1, N, 2, d)))
    k, v = rnd((1, N, 1, d), 15), rnd((1, N, 1, d), 16)
    o, lse = oracle.attn(q, k, v, causal, window, 1.0)
    vv = f64(v)[0, :, 0]
    for i in range(N):
        keys = [j for j in range(N) if visible(i, j, causal, window)]
        mean = [math.fsum(vv[j, c] for j in keys) / len(keys) for c in range(d)]
        expect_n = N if not causal else (i + 1 if window <= 0 else min(i + 1, window))
        assert len(keys) == expect_n
        for h in range(2):
            np.testing.assert_allclose(o[0, i, h], mean, rtol=0, atol=1e-14)
            assert abs(lse[0, h, i] - math.log(expect_n)) < 1e-14


def test_permutation_equivariance_no_mask():
    N, H, d = 29, 2, 16
    q, k, v = rnd((1, N, H, d), 17), rnd((1, N, H, d), 18), rnd((1, N, H, d), 19)
    o, lse = oracle.attn(q, k, v, False, 0, 0.25)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(3))
    o2, lse2 = oracle.attn(q, k[:, perm], v[:, perm], False, 0, 0.25)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-14)
    o3, lse3 = oracle.attn(q[:, perm], k, v, False, 0, 0.25)
    np.testing.assert_array_equal(o3[0], o[0][perm.numpy()])
    np.testing.assert_array_equal(lse3[0], lse[0][:, perm.numpy()])


def test_key_shift_invariance():
    """K_j <- K_j + t for every j leaves O unchanged and moves LSE_i by scale*q_i.t
    (integer-valued inputs, so the shifted keys are exact in bf16)."""
    N, d, scale = 15, 8, 0.125
    q = rnd((1, N, 1, d), 20, -3, 3)
    k = rnd((1, N, 1, d), 21, -3, 3)
    v = rnd((1, N, 1, d), 22)
    t = rnd((d,), 23, -4, 4)
    for causal in (False, True):
        o, lse = oracle.attn(q, k, v, causal, 0, scale)
        o2, lse2 = oracle.attn(q, (k.float() + t.float()).to(torch.bfloat16), v, causal, 0, scale)
        np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
        shift = scale * (f64(q)[0, :, 0] @ f64(t))
        np.testing.assert_allclose(lse2[0, 0] - lse[0, 0], shift, rtol=0, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv():
    N, Hq, Hkv, d = 33, 8, 2, 16
    q, k, v = rnd((1, N, Hq, d), 24), rnd((1, N, Hkv, d), 25), rnd((1, N, Hkv, d), 26)
    o, lse = oracle.attn(q, k, v, True, 0, 0.25)
    g = Hq // Hkv
    o2, lse2 = oracle.attn(q, k.repeat_interleave(g, dim=2), v.repeat_interleave(g, dim=2),
                           True, 0, 0.25)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    # MQA: one KV head for every query head
    o3, _ = oracle.attn(q, k[:, :, :1], v[:, :, :1], True, 0, 0.25)
    o4, _ = oracle.attn(q, k[:, :, :1].repeat_interleave(Hq, dim=2),
                        v[:, :, :1].repeat_interleave(Hq, dim=2), True, 0, 0.25)
    np.testing.assert_array_equal(o3, o4)


def test_window_edge_cases():
    N, d = 20, 8
    q, k, v = rnd((1, N, 2, d), 27), rnd((1, N, 2, d), 28), rnd((1, N, 2, d), 29)
    o1, lse1 = oracle.attn(q, k, v, True, 1, 0.3)
    np.testing.assert_array_equal(o1, f64(v))          # W=1: each token sees itself
    for h in range(2):
        for i in range(N):
            dot = math.fsum(float(a) * float(b) for a, b in zip(f64(q)[0, i, h], f64(k)[0, i, h]))
            assert abs(lse1[0, h, i] - 0.3 * dot) < 1e-13
    oc, lc = oracle.attn(q, k, v, True, 0, 0.3)
    for W in (N, N + 7):                                # W >= N is plain causal
        ow, lw = oracle.attn(q, k, v, True, W, 0.3)
        np.testing.assert_array_equal(ow, oc)
        np.testing.assert_array_equal(lw, lc)


def _single_query(qrow, keys, vals, page_size=1, scale=0.25):
    """One query over an explicit key list via the paged-decode entry (the
    query sits at the last position and sees every key)."""
    L, Hkv, d = keys.shape
    npg = (L + page_size - 1) // page_size
    pad = npg * page_size - L
    kc = torch.cat([keys, torch.zeros((pad, Hkv, d), dtype=keys.dtype)]).view(npg, page_size, Hkv, d)
    vc = torch.cat([vals, torch.zeros((pad, Hkv, d), dtype=vals.dtype)]).view(npg, page_size, Hkv, d)
    bt = torch.arange(npg, dtype=torch.int32)[None]
    return oracle.decode_paged(qrow[None], kc, vc, bt, torch.tensor([L], dtype=torch.int32), scale)


def test_split_combine_identity():
    """Flash-Decoding: attend to chunks of the keys separately and merge with
    log-sum-exp; the merge equals attention over all keys."""
    L, Hq, Hkv, d = 300, 4, 1, 16
    q, k, v = rnd((Hq, d), 30), rnd((L, Hkv, d), 31), rnd((L, Hkv, d), 32)
    o_full, lse_full = _single_query(q, k, v)
    cuts = [0, 1, 77, 128, 129, 300]
    parts = [_single_query(q, k[a:b], v[a:b]) for a, b in zip(cuts, cuts[1:])]
    o_parts = np.stack([p[0][0] for p in parts])       # [P, Hq, d]
    lse_parts = np.stack([p[1][0] for p in parts])     # [P, Hq]
    o, lse = oracle.lse_combine(o_parts, lse_parts)
    np.testing.assert_allclose(o, o_full[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_full[0], rtol=0, atol=1e-12)
    # a part over no keys carries no weight
    o2, lse2 = oracle.lse_combine(np.concatenate([o_parts, np.zeros((1, Hq, d))]),
                                  np.concatenate([lse_parts, np.full((1, Hq), -np.inf)]))
    np.testing.assert_array_equal(o2, o)
    np.testing.assert_array_equal(lse2, lse)
    o3, lse3 = oracle.lse_combine(np.zeros((2, 3, 4)), np.full((2, 3), -np.inf))
    assert np.all(o3 == 0) and np.all(lse3 == -np.inf)


def test_online_recurrence_matches_page_example():
    """The page's numpy check: q in R^128, K, V of 4096x128 from
    default_rng(0), tiled online softmax with block 64 against the two-pass
    result; it prints a max difference of 1.39e-16.  Our own fp64 re-run of the
    running-max/running-sum recurrence (on the bf16-rounded inputs the oracle
    takes) must agree with the oracle to the same order."""
    spec = json.load(open(os.path.join(GOLD, "online_softmax_example.json")))
    rng = np.random.default_rng(spec["seed"])
    q = rng.standard_normal(spec["d"])
    K = rng.standard_normal((spec["n_keys"], spec["d"]))
    V = rng.standard_normal((spec["n_keys"], spec["d"]))
    qb, Kb, Vb = bf(q), bf(K), bf(V)
    qd, Kd, Vd = f64(qb), f64(Kb), f64(Vb)
    scale = 1.0 / math.sqrt(spec["d"])
    m, l, acc = -np.inf, 0.0, np.zeros(spec["d"])
    for i in range(0, spec["n_keys"], spec["block"]):
        s = Kd[i:i + spec["block"]] @ qd * scale
        m_new = max(m, s.max())
        a = math.exp(m - m_new)
        p = np.exp(s - m_new)
        l = l * a + p.sum()
        acc = acc * a + p @ Vd[i:i + spec["block"]]
        m = m_new
    tiled = acc / l
    o, lse = _single_query(qb[None], Kb[:, None], Vb[:, None], page_size=16, scale=scale)
    diff = np.abs(o[0, 0] - tiled).max()
    assert diff <= 100 * spec["printed_max_abs_diff"], diff
    assert abs(lse[0, 0] - (m + math.log(l))) < 1e-12


def test_paged_decode_equals_contiguous_last_row():
    lens = [1, 15, 16, 17, 50]
    Hq, Hkv, d, ps = 4, 2, 16, 16
    import workloads
    inp = workloads.paged(lens=lens, Hq=Hq, Hkv=Hkv, d=d, page_size=ps, seed=5,
                          poison=True, spare_pages=2)
    o, lse = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                 inp.seq_lens, inp.scale)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(lse))
    for s, L in enumerate(lens):
        pages = inp.block_table[s, :(L + ps - 1) // ps].long()
        kk = inp.k_cache[pages].reshape(-1, Hkv, d)[:L]
        vv = inp.v_cache[pages].reshape(-1, Hkv, d)[:L]
        qq = torch.zeros((L, Hq, d), dtype=torch.bfloat16)
        qq[L - 1] = inp.q[s]
        oc, lc = oracle.attn(qq[None], kk[None], vv[None], True, 0, inp.scale)
        np.testing.assert_array_equal(o[s], oc[0, L - 1])
        np.testing.assert_array_equal(lse[s], lc[0, :, L - 1])


def test_varlen_equals_per_sequence_dense():
    import workloads
    inp = workloads.varlen(lens=[5, 1, 40, 17], Hq=4, Hkv=2, d=16, causal=True,
                           window=6, seed=3)
    o, lse = oracle.attn_varlen(inp.q, inp.k, inp.v, inp.cu_seqlens, True, 6, inp.scale)
    cu = inp.cu_seqlens.tolist()
    for s in range(len(inp.lens)):
        a, b = cu[s], cu[s + 1]
        od, ld = oracle.attn(inp.q[a:b][None], inp.k[a:b][None], inp.v[a:b][None],
                             True, 6, inp.scale)
        np.testing.assert_array_equal(o[a:b], od[0])
        np.testing.assert_array_equal(lse[:, a:b], ld[0])
    # sampled rows agree with the full run
    rows = [0, 4, 5, 6, 45, 62]
    orr, lrr = oracle.attn_varlen(inp.q, inp.k, inp.v, inp.cu_seqlens, True, 6,
                                  inp.scale, rows=rows)
    np.testing.assert_array_equal(orr, o[rows])
    np.testing.assert_array_equal(lrr, lse[:, rows].T)


def test_bad_arguments_rejected():
    q = bf(np.zeros((1, 4, 3, 8)))
    k = bf(np.zeros((1, 4, 2, 8)))
    with pytest.raises(ValueError):
        oracle.attn(q, k, k, False, 0, 1.0)   # Hq % Hkv != 0
