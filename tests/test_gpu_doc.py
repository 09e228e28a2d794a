"""GPU parity of the document-masked prefill (fa_fwd_doc) against the fp64
oracle, through the C ABI.  Same tolerances as the prefill (tests/parity.py)."""
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


def doc_ids(B, N, ndocs, seed, contiguous=False):
    g = torch.Generator("cpu").manual_seed(seed)
    if contiguous:
        cuts = torch.sort(torch.randint(1, N, (B, ndocs - 1), generator=g)).values
        ids = torch.zeros((B, N), dtype=torch.int32)
        for b in range(B):
            for c in cuts[b].tolist():
                ids[b, c:] += 1
        return ids
    return torch.randint(0, ndocs, (B, N), generator=g, dtype=torch.int32)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("N,causal,window,ndocs", [
    (300, True, 0, 3), (257, False, 0, 2), (640, True, 100, 4), (129, True, 0, 1),
    (513, True, 0, 40)])
def test_interleaved_documents(fa, N, causal, window, ndocs, d):
    inp = workloads.dense(2, 4, 2, N, d, causal=causal, window=window, seed=N + ndocs)
    doc = doc_ids(2, N, ndocs, seed=N)
    o, lse = fa.fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), causal, window, inp.scale,
                    doc_ids=doc.cuda())
    assert fa.check_device_error() == 0
    o_ref, lse_ref = oracle.attn_doc(inp.q, inp.k, inp.v, doc, causal, window, inp.scale)
    compare(o, o_ref, lse, lse_ref, f"doc N={N} causal={causal} W={window} docs={ndocs} d={d}")


def test_contiguous_documents_equal_varlen(fa):
    B, N = 1, 700
    inp = workloads.dense(B, 8, 2, N, 128, causal=True, seed=7)
    doc = doc_ids(B, N, 5, seed=7, contiguous=True)
    q, k, v = inp.q.cuda(), inp.k.cuda(), inp.v.cuda()
    o, lse = fa.fwd(q, k, v, True, 0, inp.scale, doc_ids=doc.cuda())
    lens = torch.bincount(doc[0].long()).tolist()
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32).cuda()
    o2, lse2 = fa.fwd_varlen(q[0], k[0], v[0], cu, max(lens), True, 0, inp.scale)
    assert (o[0].float() - o2.float()).abs().max().item() <= 2e-2
    assert (lse[0] - lse2).abs().max().item() <= 1e-3


def test_gqa4k_shape_documents(fa):
    """The 4k GQA shape with 64 interleaved documents: sampled rows."""
    inp = workloads.make("gqa4k", seed=0)
    B, N, Hq, d = inp.q.shape
    doc = doc_ids(B, N, 64, seed=0)
    o, lse = fa.fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), True, 0, inp.scale,
                    doc_ids=doc.cuda())
    assert fa.check_device_error() == 0
    g = torch.Generator("cpu").manual_seed(1)
    rows = sorted(set([0, 1, 127, 128, 2047, 4095] + torch.randint(0, N, (20,), generator=g).tolist()))
    o_ref, lse_ref = oracle.attn_doc(inp.q, inp.k, inp.v, doc, True, 0, inp.scale,
                                     rows=[(0, i) for i in rows])
    compare(o[0, rows], o_ref, lse[0][:, rows].T, lse_ref, "doc gqa4k")
