"""GPU parity of the chunked prefill over a paged cache (fa_fwd_paged) against
the fp64 oracle, through the C ABI.  Same tolerances as the prefill
(tests/parity.py).  Unused cache slots and spare pages are NaN-poisoned."""
import math

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


def run(fa, w, causal=True, window=0, sinks=None, out_dtype=torch.bfloat16):
    o, lse = fa.fwd_paged(w.q.cuda(), w.k_cache.cuda(), w.v_cache.cuda(), w.block_table.cuda(),
                          w.cu_seqlens_q.cuda(), w.seq_lens_k.cuda(), w.max_seqlen_q, causal,
                          window, w.scale, sinks=None if sinks is None else sinks.cuda(),
                          out_dtype=out_dtype)
    assert fa.check_device_error() == 0
    return o, lse


CASES = [
    ([300], [300]), ([300], [1]), ([513], [37]), ([1000, 17, 129, 256], [200, 17, 1, 128]),
    ([77, 0, 40], [5, 0, 40]), ([2048, 700], [512, 300]), ([16, 31, 33], [16, 1, 33]),
]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("lens_k,lens_q", CASES)
def test_chunks(fa, lens_k, lens_q, d):
    w = workloads.paged_prefill(lens_k, lens_q, Hq=8, Hkv=2, d=d, seed=sum(lens_k) + d,
                                poison=True, spare_pages=2)
    o, lse = run(fa, w)
    o_ref, lse_ref = oracle.prefill_paged(w.q, w.k_cache, w.v_cache, w.block_table,
                                          w.cu_seqlens_q, w.seq_lens_k, True, 0, w.scale)
    compare(o, o_ref, lse, lse_ref, f"paged lens_k={lens_k} lens_q={lens_q} d={d}")


@pytest.mark.parametrize("causal,window", [(False, 0), (True, 100), (True, 1)])
def test_masks(fa, causal, window):
    w = workloads.paged_prefill([900, 260], [300, 260], Hq=4, Hkv=4, d=128, seed=window,
                                poison=True)
    o, lse = run(fa, w, causal, window)
    o_ref, lse_ref = oracle.prefill_paged(w.q, w.k_cache, w.v_cache, w.block_table,
                                          w.cu_seqlens_q, w.seq_lens_k, causal, window, w.scale)
    compare(o, o_ref, lse, lse_ref, f"paged causal={causal} W={window}")


def test_sinks_and_fp32_out(fa):
    w = workloads.paged_prefill([400, 130], [100, 130], Hq=8, Hkv=2, d=128, seed=3, poison=True)
    z = torch.randn(8, generator=torch.Generator("cpu").manual_seed(3)) * 2.0
    z[2] = -math.inf
    o, lse = run(fa, w, sinks=z, out_dtype=torch.float32)
    o_ref, lse_ref = oracle.prefill_paged(w.q, w.k_cache, w.v_cache, w.block_table,
                                          w.cu_seqlens_q, w.seq_lens_k, True, 0, w.scale,
                                          sinks=z.double().numpy())
    compare(o, o_ref, lse, lse_ref, "paged sinks")


def test_whole_sequence_chunk_equals_varlen(fa):
    """L_q = L_k with the cache holding the sequence: the same tiles and the
    same arithmetic as the packed prefill, so the results are identical."""
    lens = [700, 129, 1]
    w = workloads.paged_prefill(lens, lens, Hq=8, Hkv=2, d=128, seed=11)
    o, lse = run(fa, w)
    # the same K/V, packed contiguously
    ks, vs = [], []
    for s, L in enumerate(lens):
        rows_k, rows_v = [], []
        for p in range(-(-L // 16)):
            pg = int(w.block_table[s, p])
            rows_k.append(w.k_cache[pg]); rows_v.append(w.v_cache[pg])
        ks.append(torch.cat(rows_k)[:L]); vs.append(torch.cat(rows_v)[:L])
    k, v = torch.cat(ks).cuda(), torch.cat(vs).cuda()
    o2, lse2 = fa.fwd_varlen(w.q.cuda(), k, v, w.cu_seqlens_q.cuda(), max(lens), True, 0, w.scale)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_bad_lengths_reported(fa):
    """A chunk longer than its sequence's keys is skipped and reported."""
    w = workloads.paged_prefill([64, 100], [32, 100], Hq=2, Hkv=2, d=64, seed=2)
    sl = w.seq_lens_k.clone()
    sl[1] = 50                     # L_q = 100 > 50 keys
    o = torch.zeros((w.q.shape[0], 2, 64), dtype=torch.bfloat16, device="cuda")
    fa.fwd_paged(w.q.cuda(), w.k_cache.cuda(), w.v_cache.cuda(), w.block_table.cuda(),
                 w.cu_seqlens_q.cuda(), sl.cuda(), w.max_seqlen_q, True, 0, w.scale, out=o)
    assert fa.check_device_error() == fa.FA_ERR_INVALID_ARG
    assert torch.all(o[32:] == 0)                       # sequence 1 untouched
    o_ref, _ = oracle.prefill_paged(w.q[:32], w.k_cache, w.v_cache, w.block_table[:1],
                                    w.cu_seqlens_q[:2], w.seq_lens_k[:1], True, 0, w.scale)
    compare(o[:32], o_ref, what="paged valid sequence")


def test_long_context_chunk(fa):
    """8 sequences of 8K-16K cached tokens, chunks of 512-2048 new tokens
    (Hq=32, Hkv=8, d=128): sampled rows against the oracle."""
    g = torch.Generator("cpu").manual_seed(5)
    lens_q = workloads.draw_lengths(8, 512, 2048, g)
    lens_k = [q + c for q, c in zip(lens_q, workloads.draw_lengths(8, 8192, 14336, g))]
    w = workloads.paged_prefill(lens_k, lens_q, Hq=32, Hkv=8, d=128, seed=5)
    o, lse = run(fa, w)
    cu = w.cu_seqlens_q.tolist()
    rows = sorted(set([cu[s] for s in range(8)] + [cu[s + 1] - 1 for s in range(8)] +
                      torch.randint(0, cu[-1], (24,), generator=g).tolist()))
    # oracle on the sampled rows only: one-row chunks at those positions
    for t in rows:
        s = max(i for i in range(8) if cu[i] <= t)
        pos = lens_k[s] - lens_q[s] + (t - cu[s])
        qs = w.q[t:t + 1]
        o_ref, lse_ref = oracle.prefill_paged(qs, w.k_cache, w.v_cache, w.block_table[s:s + 1],
                                              torch.tensor([0, 1], dtype=torch.int32),
                                              torch.tensor([pos + 1], dtype=torch.int32),
                                              True, 0, w.scale)
        compare(o[t:t + 1], o_ref, lse[:, t:t + 1], lse_ref, f"long chunk row {t}")
