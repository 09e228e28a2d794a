"""Pins for the oracle's document mask (FlexAttention's document masks, Ales
Analytics kernels page): key j is visible from query i only if both tokens
carry the same document id.  Pins reduce it to pinned functions: one id for
every token is plain attention; contiguous documents are the packed-sequence
(varlen) attention; an interleaved layout equals, per document, attention over
that document's tokens gathered in order."""
import numpy as np
import pytest
import torch

import oracle


def rnd(shape, seed):
    g = torch.Generator("cpu").manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


@pytest.mark.parametrize("causal,window", [(0, 0), (1, 0), (1, 9)])
def test_single_document_is_plain(causal, window):
    q, k, v = rnd((2, 40, 4, 16), 1), rnd((2, 40, 2, 16), 2), rnd((2, 40, 2, 16), 3)
    doc = torch.full((2, 40), 7, dtype=torch.int32)
    o, l = oracle.attn_doc(q, k, v, doc, causal, window, 0.3)
    o2, l2 = oracle.attn(q, k, v, causal, window, 0.3)
    assert np.array_equal(o, o2) and np.array_equal(l, l2)


def test_contiguous_documents_are_varlen():
    lens = [13, 1, 30, 20]
    N = sum(lens)
    q, k, v = rnd((1, N, 4, 16), 4), rnd((1, N, 2, 16), 5), rnd((1, N, 2, 16), 6)
    doc = torch.tensor(np.repeat(np.arange(len(lens)), lens), dtype=torch.int32).view(1, N)
    o, l = oracle.attn_doc(q, k, v, doc, True, 0, 0.3)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    o2, l2 = oracle.attn_varlen(q[0], k[0], v[0], cu, True, 0, 0.3)
    assert np.array_equal(o[0], o2) and np.array_equal(l[0], l2)


@pytest.mark.parametrize("causal", [0, 1])
def test_interleaved_documents_equal_gathered(causal):
    N = 50
    g = torch.Generator("cpu").manual_seed(8)
    doc = torch.randint(0, 3, (1, N), generator=g, dtype=torch.int32)
    q, k, v = rnd((1, N, 2, 16), 9), rnd((1, N, 1, 16), 10), rnd((1, N, 1, 16), 11)
    o, l = oracle.attn_doc(q, k, v, doc, causal, 0, 0.25)
    for dd in range(3):
        idx = torch.nonzero(doc[0] == dd).flatten()
        if idx.numel() == 0:
            continue
        og, lg = oracle.attn(q[:, idx], k[:, idx], v[:, idx], causal, 0, 0.25)
        assert np.array_equal(o[0, idx.numpy()], og[0])
        assert np.array_equal(l[0][:, idx.numpy()], lg[0])


def test_rows_subset_matches_full():
    N = 33
    g = torch.Generator("cpu").manual_seed(12)
    doc = torch.randint(0, 4, (2, N), generator=g, dtype=torch.int32)
    q, k, v = rnd((2, N, 2, 16), 13), rnd((2, N, 2, 16), 14), rnd((2, N, 2, 16), 15)
    o, l = oracle.attn_doc(q, k, v, doc, True, 0, 0.2)
    rows = [(0, 0), (0, 17), (1, 32), (1, 5)]
    orr, lr = oracle.attn_doc(q, k, v, doc, True, 0, 0.2, rows=rows)
    for r, (b, i) in enumerate(rows):
        assert np.array_equal(orr[r], o[b, i]) and np.array_equal(lr[r], l[b, :, i])
