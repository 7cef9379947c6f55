"""The N > 1 bench path on CPU: two gloo ranks, each with its own batch
(weak scaling, no data-path collective); the job time is the slowest rank's
and throughput counts every rank's steps."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    from fp4_kv_cache_append_b200 import inputs as I
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = I.small("dec_full", B=2, n=512)
        seed = bench.rank_seed(rank)
        kv = I.context_kv(wl, seed, 0, tokens=8)
        local_ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, dist, torch.device("cpu"))
        value = bench.job_throughput(world, 100, ms)
        q.put((rank, seed, kv.float().sum().item(), ms, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_weak_scaling_plumbing():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=100) for _ in procs)
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    (r0, s0, k0, ms0, v0), (r1, s1, k1, ms1, v1) = res
    assert s0 != s1 and k0 != k1                   # independent batches per rank
    assert ms0 == ms1 == 15.0                      # max over ranks
    assert v0 == v1 == pytest.approx(2 * 100 / 0.015)
