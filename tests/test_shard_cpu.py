"""The context-sharded decode step on two gloo ranks (CPU).

fp4_kv_cache_append_b200.shard runs its exchange (all-gather of the ranks'
(score, id) lists and range starts, byte-sum reduce of the compact cache to
the owner) over torch.distributed; here the per-rank compute steps are the
oracle's, so the test checks the sharding itself: the merged Top-K, the
merged pool and the owner's attention equal, exactly, the oracle's unsharded
step over the whole context.  (tests/test_gpu_shard.py runs the same phases
with the CUDA kernels on one GPU.)
"""
import os

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle

B, N, D, DI, H, H_I, K, P, W = 2, 1000, 128, 64, 4, 4, 64, 32, 32


class OracleOps:
    """The compute steps of shard.CudaOps, by the oracle on host arrays."""

    def __init__(self, K, P):
        self.K, self.P = K, P

    def local_select(self, shard, q_idx, w, q_pos):
        from fp4_kv_cache_append_b200.shard import Local
        idx, sc, pool, psc = [], [], [], []
        for b in range(shard.B):
            n = int(shard.n_entries[b])
            s = oracle.index_scores(shard, b, q_idx[b], w[b], n)
            top = oracle.topk(s, self.K)
            idx.append(top)
            sc.append(np.where(top >= 0, s[np.maximum(top, 0)], -np.inf))
            bl = oracle.block_pool(s, self.P)
            pad = np.full((n + 7) // 8 * 8, -np.inf)
            pad[:n] = s
            bm = pad.reshape(-1, 8).max(axis=1)
            pool.append(bl)
            psc.append(np.where(bl >= 0, bm[np.maximum(bl, 0)], -np.inf))
        t = lambda x, dt: torch.from_numpy(np.stack(x).astype(dt))
        return Local(t(idx, np.int32), t(sc, np.float32), t(pool, np.int32), t(psc, np.float32))

    def merge(self, scores, ids, seg_base, K):
        G, Bn, n = scores.shape
        out = np.full((Bn, K), -1, np.int32)
        for b in range(Bn):
            gid = {}
            for g in range(G):
                for i in range(n):
                    if ids[g, b, i] >= 0:
                        gid[int(ids[g, b, i]) + seg_base[g]] = float(scores[g, b, i])
            dense = np.full(max(gid) + 1 if gid else 1, -np.inf)
            for e, v in gid.items():
                dense[e] = v
            out[b] = oracle.topk(dense, K)
        return torch.from_numpy(out), None

    def gather(self, shard, lo, ids):
        Bn, Kn = ids.shape
        codes = np.zeros((Bn, Kn, shard.D // 2), np.uint8)
        scales = np.zeros((Bn, Kn, shard.D // 16), np.uint8)
        pos = np.where(ids.numpy() >= 0, np.arange(Kn)[None, :], -1).astype(np.int32)
        for b in range(Bn):
            for k in range(Kn):
                e = int(ids[b, k]) - lo
                if ids[b, k] >= 0 and 0 <= e < shard.cap:
                    codes[b, k], scales[b, k] = shard.codes[b, e], shard.scales[b, e]
        return torch.from_numpy(codes), torch.from_numpy(scales), torch.from_numpy(pos)

    def attention(self, codes, scales, shard, swa, q, q_pos, pos, scale, out):
        Bn, Kn = codes.shape[0], codes.shape[1]
        compact = oracle.MainCache(Bn, Kn, swa.D, shard.dI, 1)
        compact.codes[:], compact.scales[:] = codes.numpy(), scales.numpy()
        for b in range(Bn):
            out[b] = torch.from_numpy(oracle.attention(compact, swa, b, q[b], pos[b].numpy(), int(q_pos[b, 0]),
                                                       scale).astype(np.int16))


def _inputs():
    g = torch.Generator().manual_seed(5)
    kv = torch.randn(B, N, D, generator=g).to(torch.bfloat16)
    Wik = (torch.randn(D, DI, generator=g) / D ** 0.5).to(torch.bfloat16)
    swa_rows = torch.randn(B, N, D, generator=g).to(torch.bfloat16)
    qi = torch.randn(B, H_I, DI, generator=g).to(torch.bfloat16)
    w = torch.rand(B, H_I, generator=g)
    q = torch.randn(B, H, D, generator=g).to(torch.bfloat16)
    bits = lambda t: t.contiguous().view(torch.int16).numpy().view(np.uint16)
    return bits(kv), bits(Wik), bits(swa_rows), bits(qi), w.numpy(), bits(q)


def _cache(kv, Wik, lo, hi):
    c = oracle.MainCache(B, max(128, (hi - lo + 127) // 128 * 128), D, DI, 1)
    oracle.append(c, kv[:, lo:hi], None, Wik, None, None, np.zeros(B, np.int32), hi - lo)
    return c


def _window(swa_rows):
    sw = oracle.SwaCache(B, W, D, window=W)
    oracle.append(None, None, None, None, sw, swa_rows[:, N - W:], np.full(B, N - W, np.int32), W)
    return sw


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist
    from fp4_kv_cache_append_b200 import shard as S
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        kv, Wik, swa_rows, qi, w, qq = _inputs()
        lo, hi = S.shard_ranges(N, world, align=128)[rank]
        r = S.Rank(shard=_cache(kv, Wik, lo, hi), lo=lo)
        if rank == world - 1:
            r.swa, r.q = _window(swa_rows), qq
        out = torch.zeros(B, H, D, dtype=torch.int16)
        q_pos = torch.full((B, 1), N - 1, dtype=torch.int32)
        idx, pool = S.step_distributed(r, OracleOps(K, P), qi, w, q_pos, 0.125, out)
        q.put((rank, lo, hi, idx.numpy(), pool.numpy(), out.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_rank_sharded_step_equals_the_unsharded_step():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29600 + os.getpid() % 1000
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=280) for _ in procs), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=30)
        assert p.exitcode == 0
    (_, lo0, hi0, idx0, pool0, _), (_, lo1, hi1, idx1, pool1, out1) = res
    assert (lo0, hi0, lo1, hi1) == (0, 512, 512, N)
    np.testing.assert_array_equal(idx0, idx1)        # every rank holds the merged selection
    np.testing.assert_array_equal(pool0, pool1)
    # the unsharded step
    kv, Wik, swa_rows, qi, w, qq = _inputs()
    full = _cache(kv, Wik, 0, N)
    sw = _window(swa_rows)
    for b in range(B):
        s = oracle.index_scores(full, b, qi[b], w[b], N)
        top = oracle.topk(s, K)
        np.testing.assert_array_equal(idx1[b], top)
        np.testing.assert_array_equal(pool1[b], oracle.block_pool(s, P))
        ref = oracle.attention(full, sw, b, qq[b], top, N - 1, 0.125)
        np.testing.assert_array_equal(out1[b].view(np.uint16), ref)
