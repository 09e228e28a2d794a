"""fa_decode_paged_noalloc: paged decode for callers that cannot allocate
device memory (a host framework's memory pool owns the device, cudaMalloc's
implicit synchronisation is not allowed on the serving path, or the memory
budget is fixed at load time).  It uses the library's fixed 32 MiB device
scratch array instead of a caller workspace.

Checked through the C ABI against the workspace-taking fa_decode_paged on
two calls in a row, within the parity tolerances.  Kept in its own file,
collected last, and independent of the other tests' state."""
import pytest
import torch

import workloads
from parity import TOL_LSE_MAX, TOL_O_MAX, TOL_O_MEAN

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_io_aware_75_b200 as fa
    return fa


def _close(a, b, la, lb):
    err = (a.float() - b.float()).abs()
    assert err.max().item() <= TOL_O_MAX and err.mean().item() <= TOL_O_MEAN
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isneginf(la), torch.isneginf(lb))
    assert (la[fin] - lb[fin]).abs().max().item() <= TOL_LSE_MAX


def test_noalloc_matches_workspace_decode_twice(fa):
    cases = [dict(lens=[1, 17, 300, 1000, 4000, 0, 2048, 33], Hq=32, Hkv=8, d=128, seed=21),
             dict(lens=[5, 700, 129], Hq=16, Hkv=4, d=64, seed=22)]
    for c in cases:
        inp = workloads.paged(lens=c["lens"], Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"],
                              seed=c["seed"], poison=True, spare_pages=2)
        args = (inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
                inp.block_table.cuda(), inp.seq_lens.cuda())
        o_ref, l_ref = fa.decode_paged(*args, inp.scale)
        o, l = fa.decode_paged_noalloc(*args, inp.scale)
        assert fa.check_device_error() == 0
        _close(o, o_ref, l, l_ref)


def test_noalloc_refuses_oversize(fa):
    """A request whose split-KV scratch would exceed the fixed 32 MiB array is
    refused before anything runs."""
    need = fa.decode_workspace_bytes(64, 32, 128, 16, 2048)
    assert need > 32 << 20
    P = 1 << 20
    rc = fa.library().fa_decode_paged_noalloc(P, P, P, P, P, P, 0, 64, 100, 32, 8, 128, 16,
                                              2048, 0.1, None)
    assert rc == fa.FA_ERR_WORKSPACE


def test_noalloc_near_limit_matches_oracle(fa):
    """64 sequences x 32 query heads, d = 128, 496 pages per block-table row:
    the split-KV scratch takes 31.5 of the array's 32 MiB, and the two full-
    length sequences (first and last) write its first and last partials.
    Every row of O and LSE is compared with the fp64 oracle, on two calls in
    a row."""
    import numpy as np

    import oracle
    from parity import compare

    g = torch.Generator("cpu").manual_seed(23)
    lens = torch.randint(1, 2049, (64,), generator=g).tolist()
    lens[0] = lens[63] = 496 * 16
    inp = workloads.paged(lens=lens, Hq=32, Hkv=8, d=128, seed=23, poison=True)
    assert inp.block_table.shape[1] == 496
    need = fa.decode_workspace_bytes(64, 32, 128, 16, 496)
    assert (31 << 20) < need <= 32 << 20
    args = (inp.q.cuda(), inp.k_cache.cuda(), inp.v_cache.cuda(),
            inp.block_table.cuda(), inp.seq_lens.cuda())
    o_ref, lse_ref = oracle.decode_paged(inp.q, inp.k_cache, inp.v_cache, inp.block_table,
                                         inp.seq_lens, inp.scale)
    for _ in range(2):
        o, lse = fa.decode_paged_noalloc(*args, inp.scale)
        assert fa.check_device_error() == 0
        compare(o, o_ref, lse, lse_ref, "noalloc near the limit")
    assert np.isfinite(o_ref).all()

