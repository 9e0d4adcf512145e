"""The bench's multi-rank bookkeeping on CPU with gloo, world size 2.

With N GPUs the path runs N independent replicas (no data exchange); the only
cross-rank steps are the barrier around the timed region, the max over ranks
of the elapsed time and the sum of the units processed.  These run here with
the gloo backend on 127.0.0.1.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    assert bench.dist_env() == (rank, world, rank)
    bench.barrier(world)
    t = bench.reduce_max(10.0 + 5.0 * rank, world)   # rank 1 is the slow one
    u = bench.reduce_sum(100.0 * (rank + 1), world)  # units each rank processed
    out[rank] = (t, u)
    dist.destroy_process_group()


def test_two_rank_reductions():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert ctx is None or ctx
    assert out[0] == out[1] == (15.0, 300.0)
    # whole-job throughput = units of all ranks / slowest rank's time
    assert out[0][1] / out[0][0] == pytest.approx(20.0)
