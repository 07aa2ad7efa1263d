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


# ------------------------------------------------------------------ split copies over N GPUs
# Each rank copies only its slice of a layer blob over its own host link; an all-gather over the
# ranks assembles the whole blob (lst_split_plan / lst_set_split_copy). The plan and the assembly
# are host logic: checked here with gloo ranks on CPU tensors standing in for the pool slots.

def _blob_sizes():
    lst = pytest.importorskip("layer_streamed_qlora_streaming_b200")
    import synthetic as syn
    return {n: lst.blob_bytes(lst.make_config(syn.WORKLOADS[n])) for n in ("tiny", "llama8b", "qwen32b")}


def test_split_plan_partitions_every_blob():
    lst = pytest.importorskip("layer_streamed_qlora_streaming_b200")
    for name, blob in _blob_sizes().items():
        for world in range(1, 9):
            covered = 0
            counts = set()
            for rank in range(world):
                off, nbytes, count = lst.split_plan(blob, world, rank)
                counts.add(count)
                assert count % 256 == 0 and off == rank * count
                assert 0 <= nbytes <= count and off + nbytes <= blob
                assert covered == min(off, blob)          # slices follow each other, no gap
                covered += nbytes
            assert covered == blob and len(counts) == 1
            assert world * counts.pop() < blob + world * 256     # padding below one 256-B unit a rank


def _split_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import layer_streamed_qlora_streaming_b200 as lst
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        for name, blob in _blob_sizes().items():
            full = torch.randint(0, 256, (blob,), dtype=torch.uint8, generator=torch.Generator().manual_seed(blob))
            off, nbytes, count = lst.split_plan(blob, world, rank)
            slot = torch.full((world * count,), 0xA5, dtype=torch.uint8)   # this rank's pool slot
            slot[off:off + nbytes] = full[off:off + nbytes]                 # its host-link copy
            out = torch.empty_like(slot)
            dist.all_gather_into_tensor(out, slot[off:off + count].clone())  # the in-place all-gather
            q.put((name, rank, bool(torch.equal(out[:blob], full))))
    finally:
        dist.destroy_process_group()


def test_split_copy_assembles_the_blob_two_gloo_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = [q.get(timeout=10) for _ in range(3 * world)]
    assert len(got) == 3 * world and all(ok for _, _, ok in got)
