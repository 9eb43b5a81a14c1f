"""Multi-rank bookkeeping of bench.py on CPU with gloo (world size 2): the
reported time is the max over ranks and a rank that does no work still takes
part in the same collectives."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    import bench

    v = bench.max_over_ranks(10.0 * (rank + 1), "cpu")
    bench.barrier(None)
    out[rank] = v
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(60)
        assert p.exitcode == 0
    assert out[0] == out[1] == 20.0


def test_bench_args_defaults():
    import bench

    a = bench.parse_args([])
    assert a.gpus == 1 and a.impl == "ours" and a.steps > 0 and a.warmup >= 3
