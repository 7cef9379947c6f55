"""Context-sharded decode step over several GPUs (call order and exchange only).

DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2" and Fig. 2: the
decode cost of a long context is the Full scan over every entry; the rest of
the step works on the <= 512 selected entries.  A sequence's entries are split
by contiguous ranges over G ranks (one process per GPU):

1. every rank runs the fused scan + selection on its range
   (``csa2_index_topk`` with the selected scores): a local Top-K and a local
   pool of blocks, each as (score, id) lists;
2. one all-gather of those lists; every rank merges them with
   ``csa2_topk_merge`` (exact: each global Top-K entry is in its own range's
   Top-K, each global pool block in its range's pool);
3. every rank copies the merged selection's entries it holds into a compact
   cache (``csa2_gather_entries``: zeros where another rank holds the entry);
   a byte-sum reduce to the owner (the rank holding the newest entries and the
   window) assembles the cache the selection points into;
4. the owner runs ``csa2_sparse_attn_decode`` on it with its window rows.

Remote entries cross the link once, into the owner's memory, before any
kernel reads them.  The arithmetic is in libcsa2; this module holds buffers,
the order of the calls and the collectives (``torch.distributed``).  The
compute steps are the methods of ``CudaOps``; ``step_emulated`` runs all
ranks' phases in one process on one GPU (the exchange is a concatenation).
"""
from __future__ import annotations

import dataclasses

import torch

from . import csa2 as C


def shard_ranges(n_entries: int, world: int, align: int = 128):
    """Contiguous entry ranges [lo, hi) per rank, starts aligned to `align`
    entries (whole 8-entry pool blocks; cache capacities stay multiples of
    128); the last rank takes the remainder (and the newest entries)."""
    per = (n_entries + world - 1) // world
    per = (per + align - 1) // align * align
    out = []
    for r in range(world):
        lo = min(r * per, n_entries)
        hi = min(lo + per, n_entries) if r < world - 1 else n_entries
        out.append((lo, hi))
    return out


@dataclasses.dataclass
class Local:
    """One rank's selection: [B][K] ids and scores, [B][P] pool ids and maxima."""
    idx: torch.Tensor
    scores: torch.Tensor
    pool: torch.Tensor | None
    pool_scores: torch.Tensor | None


class CudaOps:
    """The compute steps, as libcsa2 calls on the current CUDA device."""

    def __init__(self, K: int, P: int):
        self.K, self.P = K, P

    def local_select(self, shard: C.MainCache, q_idx, w, q_pos) -> Local:
        B, K, P = shard.B, self.K, self.P
        dev = shard.codes.device
        scores = torch.empty(B, shard.cap, dtype=torch.float32, device=dev)
        idx = torch.empty(B, K, dtype=torch.int32, device=dev)
        sc = torch.empty(B, K, dtype=torch.float32, device=dev)
        pool = torch.empty(B, P, dtype=torch.int32, device=dev) if P else None
        psc = torch.empty(B, P, dtype=torch.float32, device=dev) if P else None
        C.csa2_index_topk(shard, q_idx, w, q_pos, scores, K, idx, P_out=P, out_pool=pool, out_scores=sc,
                          out_pool_scores=psc)
        return Local(idx, sc, pool, psc)

    def merge(self, scores, ids, seg_base, K):
        G, B, _ = scores.shape
        out = torch.empty(B, K, dtype=torch.int32, device=scores.device)
        osc = torch.empty(B, K, dtype=torch.float32, device=scores.device)
        C.csa2_topk_merge(scores, ids, seg_base, K, out, osc)
        return out, osc

    def gather(self, shard: C.MainCache, lo: int, ids):
        B, K = ids.shape
        kcap = (K + 127) // 128 * 128
        codes = torch.empty(B, kcap, shard.D // 2, dtype=torch.uint8, device=ids.device)
        scales = torch.empty(B, kcap, shard.D // 16, dtype=torch.uint8, device=ids.device)
        codes[:, K:].zero_()
        scales[:, K:].zero_()
        pos = torch.empty(B, K, dtype=torch.int32, device=ids.device)
        C.csa2_gather_entries(shard, lo, ids, codes, scales, pos)
        return codes, scales, pos

    def attention(self, codes, scales, shard: C.MainCache, swa: C.SwaCache, q, q_pos, pos, scale, out):
        B, kcap = codes.shape[0], codes.shape[1]
        compact = C.MainCache(B, kcap, swa.D, shard.d_I, 1, device=codes.device)
        compact.codes, compact.scales = codes, scales
        compact.n_entries.fill_(kcap)
        ws = C.workspace(C.csa2_attn_workspace_size(B, 1, q.shape[-2], swa.D, pos.shape[-1], swa.window),
                         codes.device)
        C.csa2_sparse_attn_decode(compact, swa, q, q_pos, pos.view(B, 1, -1), scale, out, ws=ws)


@dataclasses.dataclass
class Rank:
    """One rank's state for a step: its shard (entries lo .. lo + n of each
    sequence), and on the owner the window cache and the attention query."""
    shard: C.MainCache
    lo: int
    swa: C.SwaCache | None = None
    q: torch.Tensor | None = None


def _merge_all(ops, gathered_scores, gathered_ids, bases, K):
    return ops.merge(gathered_scores, gathered_ids, bases, K)


def step_emulated(ranks, ops, q_idx, w, q_pos, scale, out, owner=None):
    """All ranks' phases in one process (one GPU): the all-gather is a
    concatenation and the reduce a byte sum.  Returns (idx, pool)."""
    owner = len(ranks) - 1 if owner is None else owner
    locs = [ops.local_select(r.shard, q_idx, w, q_pos) for r in ranks]
    bases = [r.lo for r in ranks]
    idx, _ = _merge_all(ops, torch.stack([l.scores for l in locs]), torch.stack([l.idx for l in locs]), bases, ops.K)
    pool = None
    if ops.P:
        pool, _ = _merge_all(ops, torch.stack([l.pool_scores for l in locs]), torch.stack([l.pool for l in locs]),
                             [b // 8 for b in bases], ops.P)
    parts = [ops.gather(r.shard, r.lo, idx) for r in ranks]
    codes = parts[0][0].clone()
    scales = parts[0][1].clone()
    for p in parts[1:]:
        codes += p[0]          # one nonzero contributor per slot: the byte sum is the entry
        scales += p[1]
    o = ranks[owner]
    ops.attention(codes, scales, o.shard, o.swa, o.q, q_pos, parts[owner][2], scale, out)
    return idx, pool


def step_distributed(rank: Rank, ops, q_idx, w, q_pos, scale, out, group=None, owner=None):
    """This process's part of the step; every rank calls it with its own
    Rank (the same q_idx, w, q_pos everywhere).  Collectives: one all-gather
    of the selection lists (and of the pool lists), one all-gather of the
    range starts, one byte-sum reduce of the compact cache to the owner.
    Returns (idx, pool) on every rank; `out` is written on the owner."""
    import torch.distributed as dist
    G = dist.get_world_size(group)
    me = dist.get_rank(group)
    owner = G - 1 if owner is None else owner
    loc = ops.local_select(rank.shard, q_idx, w, q_pos)
    lo_t = torch.tensor([rank.lo], dtype=torch.int64, device=loc.idx.device)
    los = [torch.empty_like(lo_t) for _ in range(G)]
    dist.all_gather(los, lo_t, group=group)
    bases = [int(x.item()) for x in los]

    def gather_lists(t):
        parts = [torch.empty_like(t) for _ in range(G)]
        dist.all_gather(parts, t.contiguous(), group=group)
        return torch.stack(parts)

    idx, _ = _merge_all(ops, gather_lists(loc.scores), gather_lists(loc.idx), bases, ops.K)
    pool = None
    if ops.P:
        pool, _ = _merge_all(ops, gather_lists(loc.pool_scores), gather_lists(loc.pool), [b // 8 for b in bases],
                             ops.P)
    codes, scales, pos = ops.gather(rank.shard, rank.lo, idx)
    dist.reduce(codes, dst=owner, op=dist.ReduceOp.SUM, group=group)
    dist.reduce(scales, dst=owner, op=dist.ReduceOp.SUM, group=group)
    if me == owner:
        ops.attention(codes, scales, rank.shard, rank.swa, rank.q, q_pos, pos, scale, out)
    return idx, pool
