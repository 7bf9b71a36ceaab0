"""Multi-rank host logic on CPU (gloo, world size 2): the benchmark's
replica timing takes the maximum over ranks and every rank takes the same
collective steps."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    got = bench.dist_env()
    m = bench.reduce_max(10.0 + 5.0 * rank)          # per-rank elapsed ms
    bench.barrier()
    m2 = bench.reduce_max(-1.0 * rank)
    q.put((rank, got, m, m2))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, world_got, lr), m, m2 in res:
        assert (r, world_got, lr) == (rank, 2, rank)
        assert m == 15.0          # max over ranks of 10, 15
        assert m2 == 0.0


def test_reduce_max_single_process_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
