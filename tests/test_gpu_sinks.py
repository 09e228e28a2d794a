"""GPU parity of the learned attention sink (fa_fwd_sinks, fa_fwd_varlen_sinks,
fa_decode_paged_sinks) against the fp64 oracle, through the C ABI.  Same
tolerances as plain attention (tests/parity.py)."""
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


def sink_logits(Hq, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    z = torch.randn(Hq, generator=g, dtype=torch.float32) * 2.0
    z[0] = -math.inf          # one head without a sink
    if Hq > 2:
        z[1] = 12.0           # one sink that dominates the row
    return z


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,causal,window", [(200, False, 0), (300, True, 0), (700, True, 129)])
def test_prefill_sinks(fa, N, causal, window, d):
    inp = workloads.dense(1, 4, 2, N, d, causal=causal, window=window, seed=N)
    z = sink_logits(4, N)
    o, lse = fa.fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), causal, window, inp.scale,
                    sinks=z.cuda())
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.attn_sinks(inp.q, inp.k, inp.v, z.double().numpy(), causal, window,
                                       inp.scale)
    compare(o, o_ref, lse, lse_ref, f"sinks N={N} causal={causal} W={window} d={d}")


def test_prefill_minus_inf_sinks_equal_plain(fa):
    inp = workloads.dense(1, 4, 2, 333, 128, causal=True, seed=9)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    o1, l1 = fa.fwd(q, k, v, True, 0, inp.scale)
    o2, l2 = fa.fwd(q, k, v, True, 0, inp.scale,
                    sinks=torch.full((4,), -math.inf, device="cuda"))
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_varlen_sinks(fa):
    inp = workloads.varlen(lens=[100, 0, 257, 31], Hq=8, Hkv=2, d=128, causal=True, seed=4)
    z = sink_logits(8, 4)
    o, lse = fa.fwd_varlen(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), inp.cu_seqlens.cuda(),
                           inp.max_seqlen, True, 0, inp.scale, sinks=z.cuda())
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.attn_varlen_sinks(inp.q, inp.k, inp.v, inp.cu_seqlens,
                                              z.double().numpy(), True, 0, inp.scale)
    compare(o, o_ref, lse, lse_ref, "varlen sinks")


def test_decode_sinks(fa):
    inp = workloads.paged(lens=[1, 0, 17, 300, 5000], Hq=32, Hkv=8, d=128, seed=6)
    z = sink_logits(32, 6)
    o, lse = fa.decode_paged(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                             inp.block_table.cuda(), inp.seq_lens.cuda(), inp.scale,
                             sinks=z.cuda())
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.decode_paged_sinks(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                               inp.seq_lens, z.double().numpy(), inp.scale)
    compare(o, o_ref, lse, lse_ref, "decode sinks")
    # the empty sequence: O = 0, LSE = z_h
    assert torch.all(o[1] == 0)
    fin = torch.isfinite(z)
    assert torch.allclose(lse[1].cpu()[fin], z[fin])
