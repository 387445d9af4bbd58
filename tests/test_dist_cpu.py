"""Rank-level logic of the data-parallel replicas, on CPU with gloo (world size 2):
the adapter-gradient all-reduce and the max-over-ranks step time used by bench.py."""

import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w = bench.init_dist("gloo")
    assert (r, w) == (rank, world)
    dq = torch.full((3, 5, 7), float(rank + 1))
    bench.allreduce_grad(dq)
    t = bench.max_over_ranks(10.0 + rank, torch.device("cpu"))
    q.put((rank, float(dq.sum()), dq.numel(), t))
    dist.barrier()
    dist.destroy_process_group()


def test_allreduce_and_max_over_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, s, n, t in res:
        assert s == 3.0 * n          # 1 + 2 on every element
        assert t == 11.0             # the slower rank's time
