"""The multi-rank plumbing of bench.py on CPU: two gloo ranks, the gradient average (the only
exchange of data-parallel replicas, applied by every replica's deferred AdamW update), max-over-ranks
timing and the whole-job throughput."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.full((1000,), float(rank + 1))
        bench.allreduce_grads(g, dist)
        # uneven length, values whose sum rounds: every rank gets the fixed-order mean, same bytes
        gen = torch.Generator().manual_seed(7)
        all_g = [torch.randn(1001, generator=gen) * 10 ** k for k in range(world)]
        mine = all_g[rank].clone()
        bench.allreduce_grads(mine, dist)
        ref = all_g[0].clone()
        for k in range(1, world):
            ref += all_g[k]
        ref /= world
        q.put(("mean", rank, mine.numpy().tobytes() == ref.numpy().tobytes()))
        ms = bench.max_over_ranks(100.0 + 50.0 * rank, dist, "cpu")
        thr = bench.job_throughput(world, 2048, 10, ms)
        q.put((rank, float(g[0]), float(g[-1]), ms, thr))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = [q.get(timeout=10) for _ in range(2 * world)]
    assert all(ok for tag, _, ok in (x for x in got if x[0] == "mean"))
    res = sorted(x for x in got if x[0] != "mean")
    for rank, g0, g1, ms, thr in res:
        assert g0 == g1 == 1.5            # mean of 1 and 2 on both ranks
        assert ms == 150.0                # the slowest rank
        assert abs(thr - 2 * 2048 * 10 / 0.150) < 1e-6
