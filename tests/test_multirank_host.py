"""The N>1 host logic of bench.py on CPU: two gloo ranks, each with its own
seeded problem, agree on the max-over-ranks timing used for the reported
throughput.  (No data-path collective exists: ranks run independent
problems.)"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    import workloads
    w, r, _ = bench.dist_env()
    assert (w, r) == (world, rank)
    seed = bench.rank_seed(0, rank)
    inp = workloads.dense(1, 2, 1, 64, 64, causal=True, seed=seed)
    local_ms = [1.0 + rank, 5.0 - rank]
    mx = bench.max_over_ranks(local_ms)
    out[rank] = (mx, float(inp.q.float().sum()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == [2.0, 5.0]
    assert out[0][1] != out[1][1]          # independent problems per rank


def test_single_process_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
