"""GPU parity of paged split-KV decode (fa_decode_paged) against the fp64
oracle, through the C ABI."""
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


def run(fa, inp, **kw):
    o, lse = fa.decode_paged(inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                             inp.block_table.cuda(), inp.seq_lens.cuda(), inp.scale, **kw)
    assert fa.check_device_error() == 0
    return o, lse


def ref(inp):
    return oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                               inp.seq_lens, inp.scale)


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (32, 8, 64), (8, 8, 128), (16, 8, 128),
                                      (32, 1, 128), (12, 4, 64), (64, 8, 128)])
def test_small(fa, Hq, Hkv, d):
    lens = [1, 15, 16, 17, 255, 256, 257, 1000, 4097, 40]
    inp = workloads.paged(lens=lens, Hq=Hq, Hkv=Hkv, d=d, seed=Hq + Hkv + d, poison=True,
                          spare_pages=3)
    o, lse = run(fa, inp)
    o_ref, lse_ref = ref(inp)
    compare(o, o_ref, lse, lse_ref, f"decode Hq={Hq} Hkv={Hkv} d={d}")


def test_empty_sequence(fa):
    inp = workloads.paged(lens=[0, 33, 0], Hq=8, Hkv=2, d=128, seed=1)
    o, lse = run(fa, inp)
    assert torch.all(o[0] == 0) and torch.all(o[2] == 0)
    assert torch.all(torch.isneginf(lse[0])) and torch.all(torch.isneginf(lse[2]))
    o_ref, lse_ref = ref(inp)
    compare(o[1:2], o_ref[1:2], lse[1:2], lse_ref[1:2], "decode empty")


def test_block_table_permutation_invariance(fa):
    """The same logical cache stored under a different page permutation gives
    bit-identical results."""
    inp = workloads.paged(lens=[700, 31, 2049], Hq=32, Hkv=8, d=128, seed=4)
    o1, l1 = run(fa, inp)
    g = torch.Generator().manual_seed(9)
    P = inp.k_cache.shape[0]
    perm = torch.randperm(P, generator=g)           # new slot of old page i = perm[i]
    kc2 = torch.empty_like(inp.k_cache)
    vc2 = torch.empty_like(inp.v_cache)
    kc2[perm] = inp.k_cache
    vc2[perm] = inp.v_cache
    bt2 = perm[inp.block_table.long()].to(torch.int32)
    inp2 = workloads.Paged(inp.q, kc2, vc2, bt2, inp.seq_lens, inp.page_size, inp.scale)
    o2, l2 = run(fa, inp2)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_decode_matches_prefill_last_row(fa):
    """Decode of a sequence's last token agrees with the causal prefill's last
    row on the same keys (two different kernels, same definition)."""
    L, Hq, Hkv, d = 1000, 32, 8, 128
    inp = workloads.paged(lens=[L], Hq=Hq, Hkv=Hkv, d=d, seed=12)
    od, ld = run(fa, inp)
    pages = inp.block_table[0, :(L + 15) // 16].long()
    kk = inp.k_cache[pages].reshape(-1, Hkv, d)[:L]
    vv = inp.v_cache[pages].reshape(-1, Hkv, d)[:L]
    g = torch.Generator().manual_seed(3)
    qq = torch.randn((L, Hq, d), generator=g).to(torch.bfloat16)
    qq[L - 1] = inp.q[0]
    op, lp = fa.fwd(qq[None].cuda(), kk[None].cuda().contiguous(), vv[None].cuda().contiguous(),
                    True, 0, inp.scale)
    diff = (op[0, L - 1].float() - od[0].float()).abs().max().item()
    assert diff <= 2e-2
    assert (lp[0, :, L - 1] - ld[0]).abs().max().item() <= 1e-3


def test_full_size_decode64(fa):
    """64 sequences, KV lengths uniform in [4096, 32768], 16-token pages under
    a random permutation: the whole output against the oracle."""
    inp = workloads.make("decode64", seed=0)
    o, lse = run(fa, inp)
    o_ref, lse_ref = ref(inp)
    compare(o, o_ref, lse, lse_ref, "decode64")
