"""bench.py's multi-rank plumbing on CPU with gloo, world size 2: the timing
reduction is a max over ranks, barriers complete, and every rank draws its own
shard of the global batch (weak scaling: no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    from harness.inputs import make_qkv
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, _ = bench.dist_env()
        bench.barrier(w)
        got = bench.max_over_ranks(10.0 + 3 * rank, w, torch.device("cpu"))
        q, _, _ = make_qkv(1, 2, 2, 16, 64, 1 + 1000 * rank)
        checksum = float(q.float().sum())
        bench.barrier(w)
        queue.put((rank, r, got, checksum))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_timing_reduction_and_shards():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = sorted(queue.get(timeout=90) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    assert [r[1] for r in results] == [0, 1]
    assert all(r[2] == 13.0 for r in results)          # max over ranks
    assert results[0][3] != results[1][3]               # distinct shards
