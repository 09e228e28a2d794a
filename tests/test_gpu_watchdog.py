"""The device-side watchdog: a kernel wait that can never complete gives up
after about a second, records FA_ERR_TIMEOUT, and leaves the CUDA context
usable for the next call (no trap, no fault, no hang)."""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fa():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import exact_io_aware_75_b200 as fa
    return fa


def test_wait_runs_out_and_context_survives(fa):
    assert fa.check_device_error() == fa.FA_OK
    t0 = time.time()
    assert fa.selftest_watchdog() == fa.FA_OK
    assert fa.check_device_error() == fa.FA_ERR_TIMEOUT     # waits for the kernel
    elapsed = time.time() - t0
    assert 0.2 < elapsed < 10.0
    assert fa.check_device_error() == fa.FA_OK              # the word was cleared
    # the context still works: a normal call gives correct results
    inp = workloads.dense(1, 2, 2, 200, 64, causal=True, seed=4)
    o, lse = fa.fwd(inp.q.cuda(), inp.k.cuda(), inp.v.cuda(), True, 0, inp.scale)
    assert fa.check_device_error() == fa.FA_OK
    o_ref, _ = oracle.attn(inp.q, inp.k, inp.v, True, 0, inp.scale)
    assert np.abs(o.float().cpu().double().numpy() - o_ref).max() < 2e-2
