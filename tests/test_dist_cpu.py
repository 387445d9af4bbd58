"""Rank-level logic of the data-parallel replicas, on CPU with gloo (world size 2):
the adapter-gradient all-reduce and the max-over-ranks step time used by bench.py,
and the partitioning itself -- a batch split by tokens over the replicas, each
rank's adapter backward summed by the same all-reduce, gives the whole batch's
dQ, and the ranks' dX rows concatenate to the whole batch's dX (the float64
oracle on every rank)."""

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


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import numpy as np
    import bench
    from gen import LinearSpec, make_linear_case
    from npcase import linear_np
    from oracle import oft_ref
    from oracle.codecs import bf16_bits_to_f64
    bench.init_dist("gloo")
    spec = LinearSpec("dp", M=37, K=64, splits=(24, 16, 8), fmt="int4", group=32, b=16, q_sigma=0.1,
                      backward=True, seed=9)
    c = linear_np(make_linear_case(spec))
    Wt = oft_ref.weight_t(c)
    R = oft_ref.rotations(c["Q"], spec.b)
    X, dY = bf16_bits_to_f64(c["X"]), bf16_bits_to_f64(c["dY"])
    t0, t1 = bench.token_shard(spec.M, rank, world)
    dX_r, dq_r = oft_ref.linear_bwd(dY[t0:t1], X[t0:t1], Wt, spec.splits, R, spec.b)
    dq_t = torch.from_numpy(np.ascontiguousarray(dq_r))
    bench.allreduce_grad(dq_t)
    rows = [None] * world
    dist.all_gather_object(rows, (t0, t1, dX_r))
    if rank == 0:
        dX_all, dq_all = oft_ref.linear_bwd(dY, X, Wt, spec.splits, R, spec.b)
        dX_cat = np.concatenate([r[2] for r in sorted(rows, key=lambda r: r[0])])
        spans = sorted((r[0], r[1]) for r in rows)
        q.put((spans, float(np.abs(dq_t.numpy() - dq_all).max() / np.abs(dq_all).max()),
               float(np.abs(dX_cat - dX_all).max() / np.abs(dX_all).max()),
               float(np.abs(dq_r - dq_all).max() / np.abs(dq_all).max())))
    dist.barrier()
    dist.destroy_process_group()


def test_token_sharded_replicas_reproduce_the_whole_batch():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    spans, dq_err, dx_err, shard_err = q.get(timeout=10)
    assert spans == [(0, 19), (19, 37)]          # every token on exactly one rank
    assert dq_err < 1e-12                        # summed shard gradients = whole-batch dQ
    assert dx_err < 1e-12                        # dX rows are per-token
    assert shard_err > 1e-3                      # a single shard's dQ alone is not the answer


def test_token_shard_and_rank_launch():
    import bench
    for M, world in [(37, 2), (16384, 8), (5, 8), (4096, 3)]:
        spans = [bench.token_shard(M, r, world) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == M
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
        sizes = [t1 - t0 for t0, t1 in spans]
        assert max(sizes) - min(sizes) <= 1
    cmd = bench.launch_cmd(["--gpus", "4", "--steps", "3"], 4, 29555)
    i = cmd.index("torch.distributed.run")
    assert cmd[:3] == ["timeout", "-k", "60"] and cmd[i - 1] == "-m"
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and "--master-port=29555" in cmd
    assert cmd[-4:] == ["--gpus", "4", "--steps", "3"] and cmd[-5].endswith("bench.py")
