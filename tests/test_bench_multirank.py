"""bench.py's multi-rank logic on CPU with the gloo backend, world size 2:
every rank takes the same collective steps, the reported time is the max over
ranks and the whole-job value counts every rank's units."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    r, w, lr = bench.dist_env()
    assert (r, w, lr) == (rank, world, rank)
    dist.barrier()
    mx = bench.reduce_max(10.0 + 5.0 * rank, world, "cpu")
    val = bench.aggregate_throughput(100.0, world, mx)
    out[rank] = (mx, val)
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_and_aggregate_gloo_world2():
    ctx = mp.get_context("spawn")
    port = _free_port()
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1] == (15.0, 100.0 * 2 / 15.0)


def test_single_rank_paths():
    import bench
    assert bench.reduce_max(3.5, 1, "cpu") == 3.5
    assert bench.aggregate_throughput(10.0, 1, 2.0) == 5.0
