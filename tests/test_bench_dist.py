"""Multi-rank plumbing of bench.py on CPU: world size 2 over gloo.

Each rank runs an independent problem (weak scaling); the timed value is
the maximum over ranks, and every rank takes the same collective steps.
"""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from compressive_memory_transformer_sm_b200 import workloads as W

    r, wsz = bench.init_dist("gloo", timeout_s=60)
    dev = torch.device("cpu")
    bench.barrier(dev)
    got = bench.max_over_ranks(10.0 + rank, dev)
    seeds = [bench.rank_seed(W.LAYER_1B, i) for i in range(world)]
    q.put((r, wsz, got, seeds))
    dist.destroy_process_group()


def test_two_ranks_max_and_independent_seeds():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(i, 2, port, q)) for i in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, wsz, got, seeds in res:
        assert wsz == 2
        assert got == 11.0  # the slowest rank's time
        assert len(set(seeds)) == 2  # each rank draws its own problem


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
