"""Device-side checks of packed-sequence offsets (fa_fwd_varlen, fa_bwd_varlen).

cu_seqlens lives in device memory, so the host cannot validate it before the
launch.  A sequence longer than max_seqlen, or one that does not lie inside
[0, total_tokens), must be skipped -- nothing read or written for it -- and
reported through fa_check_device_error as FA_ERR_INVALID_ARG, while the
other sequences are computed as usual."""
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


def _run(fa, w, cu, max_seqlen):
    T, Hq, d = w.q.shape
    o = torch.zeros((T, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((Hq, T), dtype=torch.float32, device="cuda")
    fa.fwd_varlen(w.q.cuda(), w.k.cuda(), w.v.cuda(), cu.cuda(), max_seqlen, True, 0,
                  w.scale, out=o, lse=lse)
    return o, lse, fa.check_device_error()


def _check_seq(o, lse, w, cu, s):
    a, b = int(cu[s]), int(cu[s + 1])
    sub = torch.tensor([0, b - a], dtype=torch.int32)
    o_ref, lse_ref = oracle.attn_varlen(w.q[a:b], w.k[a:b], w.v[a:b], sub, True, 0, w.scale)
    compare(o[a:b], o_ref, lse[:, a:b], lse_ref, f"sequence {s}")


def test_sequence_longer_than_max_seqlen(fa):
    w = workloads.varlen(lens=[100, 300, 50], Hq=4, Hkv=2, d=128, seed=31)
    o, lse, err = _run(fa, w, w.cu_seqlens, 200)
    assert err == fa.FA_ERR_INVALID_ARG
    assert torch.all(o[100:400] == 0) and torch.all(lse[:, 100:400] == 0)
    _check_seq(o, lse, w, w.cu_seqlens, 0)
    _check_seq(o, lse, w, w.cu_seqlens, 2)
    # the same call with a correct max_seqlen reports nothing
    _, _, err = _run(fa, w, w.cu_seqlens, 300)
    assert err == 0


def test_offsets_past_total_or_descending(fa):
    w = workloads.varlen(lens=[100, 200], Hq=4, Hkv=2, d=64, seed=32)
    # the last offset runs past total_tokens (300): sequence 1 is skipped
    cu = torch.tensor([0, 100, 400], dtype=torch.int32)
    o, lse, err = _run(fa, w, cu, 300)
    assert err == fa.FA_ERR_INVALID_ARG
    assert torch.all(o[100:] == 0)
    _check_seq(o, lse, w, cu, 0)
    # descending offsets: sequence 1 has a negative length and is skipped;
    # sequence 0 is computed and nothing past it is written
    cu = torch.tensor([0, 100, 50], dtype=torch.int32)
    o, lse, err = _run(fa, w, cu, 200)
    assert err == fa.FA_ERR_INVALID_ARG
    assert torch.all(o[100:] == 0)
    _check_seq(o, lse, w, cu, 0)


def test_bwd_sequence_longer_than_max_seqlen(fa):
    w = workloads.varlen(lens=[130, 300], Hq=4, Hkv=2, d=128, seed=33)
    q, k, v, cu = w.q.cuda(), w.k.cuda(), w.v.cuda(), w.cu_seqlens.cuda()
    o, lse = fa.fwd_varlen(q, k, v, cu, 300, True, 0, w.scale)
    do = workloads.grad_out(tuple(q.shape), seed=33).cuda()
    assert fa.check_device_error() == 0
    dq, dk, dv = fa.bwd_varlen(q, k, v, o, do, lse, cu, 300, True, 0, w.scale)
    assert fa.check_device_error() == 0
    dq2, dk2, dv2 = fa.bwd_varlen(q, k, v, o, do, lse, cu, 200, True, 0, w.scale)
    assert fa.check_device_error() == fa.FA_ERR_INVALID_ARG
    # sequence 0 (within max_seqlen) is unaffected by the skipped one: dK, dV
    # come from one work unit per key block (same order of additions); dQ is
    # added up in L2 in an order that varies from run to run
    assert torch.equal(dk2[:130], dk[:130]) and torch.equal(dv2[:130], dv[:130])
    assert (dq2[:130].float() - dq[:130].float()).abs().max().item() <= 1e-2
