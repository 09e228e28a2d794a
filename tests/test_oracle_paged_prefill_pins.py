"""Pins for the oracle's chunked prefill over a paged cache (zenaique's
FlashAttention serving explainer, "Real-world examples": serving engines run
long prompts in chunks over a paged KV cache).  The reading: a chunk's L_q queries are the last L_q of the
sequence's seq_lens_k cached tokens.  Pins reduce it to the pinned dense
definition: the chunk's rows equal the last rows of full causal attention over
the whole sequence, whatever the page permutation; L_q = 1 is the decode."""
import math

import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def paginate(k, perm, ps=16):
    """k [L, H, d] -> pages [P, ps, H, d] laid out by the page permutation."""
    L, H, d = k.shape
    npg = -(-L // ps)
    pages = torch.zeros((len(perm), ps, H, d), dtype=k.dtype)
    for p in range(npg):
        rows = k[p * ps:(p + 1) * ps]
        pages[perm[p], :rows.shape[0]] = rows
    return pages


@pytest.mark.parametrize("Lk,Lq,window", [(37, 37, 0), (100, 20, 0), (64, 1, 0), (300, 45, 50),
                                          (16, 16, 0), (129, 128, 7)])
def test_chunk_rows_equal_last_rows_of_full_causal(Lk, Lq, window):
    Hq, Hkv, d = 4, 2, 32
    q, k, v = rnd((Lk, Hq, d), Lk), rnd((Lk, Hkv, d), Lk + 1), rnd((Lk, Hkv, d), Lk + 2)
    npg = -(-Lk // 16)
    g = torch.Generator("cpu").manual_seed(9)
    perm = torch.randperm(npg + 3, generator=g)[:npg].tolist()
    kc, vc = paginate(k, perm + [0] * 3), paginate(v, perm + [0] * 3)
    bt = torch.tensor([perm], dtype=torch.int32)
    cu = torch.tensor([0, Lq], dtype=torch.int32)
    o, lse = oracle.prefill_paged(q[Lk - Lq:], kc, vc, bt, cu, torch.tensor([Lk], dtype=torch.int32),
                                  True, window, 0.2)
    cu_full = torch.tensor([0, Lk], dtype=torch.int32)
    of, lf = oracle.attn_varlen(q, k, v, cu_full, True, window, 0.2)
    assert np.array_equal(o, of[Lk - Lq:])
    assert np.array_equal(lse, lf[:, Lk - Lq:])


def test_single_query_is_decode():
    Lk, Hq, Hkv, d = 77, 8, 2, 64
    q, k, v = rnd((1, Hq, d), 1), rnd((Lk, Hkv, d), 2), rnd((Lk, Hkv, d), 3)
    perm = [4, 0, 2, 5, 1]
    kc, vc = paginate(k, perm + [3]), paginate(v, perm + [3])
    bt = torch.tensor([perm], dtype=torch.int32)
    sl = torch.tensor([Lk], dtype=torch.int32)
    o, lse = oracle.prefill_paged(q, kc, vc, bt, torch.tensor([0, 1], dtype=torch.int32), sl)
    od, ld = oracle.decode_paged(q, kc, vc, bt, sl)
    assert np.array_equal(o, od) and np.array_equal(lse[:, 0], ld[0])


def test_batch_of_sequences_and_non_causal():
    Hq, Hkv, d = 2, 1, 16
    lens_k, lens_q = [40, 0, 18, 70], [5, 0, 18, 1]
    qs, ks, vs = [], [], []
    pages_k, pages_v, table = [], [], []
    nxt = 0
    maxp = max(-(-L // 16) for L in lens_k)
    for s, (Lk, Lq) in enumerate(zip(lens_k, lens_q)):
        k, v, q = rnd((Lk, Hkv, d), 10 + s), rnd((Lk, Hkv, d), 20 + s), rnd((Lk, Hq, d), 30 + s)
        ks.append(k); vs.append(v); qs.append(q[Lk - Lq:])
        npg = -(-Lk // 16)
        row = list(range(nxt, nxt + npg)) + [0] * (maxp - npg)
        nxt += npg
        table.append(row)
        for p in range(npg):
            pk = torch.zeros((16, Hkv, d), dtype=torch.bfloat16)
            pv = torch.zeros((16, Hkv, d), dtype=torch.bfloat16)
            pk[:min(16, Lk - 16 * p)] = k[16 * p:16 * (p + 1)]
            pv[:min(16, Lk - 16 * p)] = v[16 * p:16 * (p + 1)]
            pages_k.append(pk); pages_v.append(pv)
    kc, vc = torch.stack(pages_k), torch.stack(pages_v)
    bt = torch.tensor(table, dtype=torch.int32)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens_q)]), dtype=torch.int32)
    sl = torch.tensor(lens_k, dtype=torch.int32)
    q = torch.cat(qs)
    for causal in (True, False):
        o, lse = oracle.prefill_paged(q, kc, vc, bt, cu, sl, causal, 0, 0.3)
        for s, (Lk, Lq) in enumerate(zip(lens_k, lens_q)):
            if Lq == 0:
                continue
            qf = torch.cat([torch.zeros((Lk - Lq, Hq, d), dtype=torch.bfloat16), qs[s]])
            of, lf = oracle.attn_varlen(qf, ks[s], vs[s], torch.tensor([0, Lk], dtype=torch.int32),
                                        causal, 0, 0.3)
            a = int(cu[s])
            assert np.array_equal(o[a:a + Lq], of[Lk - Lq:])
            assert np.array_equal(lse[:, a:a + Lq], lf[:, Lk - Lq:])
