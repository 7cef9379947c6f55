"""Seeded synthetic workloads for the CSA2 step.

This module holds sizes and random draws only -- none of the method's
arithmetic -- and is the one thing the CUDA path and the oracle share.

Recipe: every tensor is drawn per sequence from its own CPU ``torch.Generator``
seeded with ``crc32("<seed>/<tensor>/<sequence>")``, so any sequence can be
regenerated alone and the draw does not depend on the device or on how many
other sequences exist.  Normal draws are ``torch.randn`` (float32) rounded to
bf16; ``w`` is ``torch.rand`` (U(0,1)); the indexer projection ``W_IK`` is
N(0, 1/D).  Planted keys (workloads "tiny" and "long") follow the recipe of
the workload table: a target u ~ N(0,1)^D per sequence, planted entries
kv = u + 0.1 N at distinct positions outside the window, query heads
q_h = u + 0.1 N, indexer query heads q^I_h = W_IK^T u + 0.1 N.
"""
from __future__ import annotations

import dataclasses
import zlib

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int          # sequences
    n: int          # context tokens per sequence at the step (prefill: prefix tokens)
    m: int          # tokens pooled per entry
    D: int          # shared KV dim
    H: int          # query heads
    H_I: int        # indexer heads
    dI: int         # indexer dim
    K: int          # Top-K
    P: int          # pool blocks produced by a Full decoder layer (0: none)
    window: int     # sliding window tokens
    mode: str       # "full" | "group" | "prefill" | "long"
    T: int = 1      # new tokens per sequence in the step
    n_reuse: int = 0
    planted: int = 0

    @property
    def first_new(self) -> int:
        """Position of the first token appended by the step.  Decode
        workloads count the step's token in n; prefill appends T tokens
        after an n-token prefix."""
        return self.n if self.mode == "prefill" else self.n - self.T

    @property
    def total_tokens(self) -> int:
        return self.first_new + self.T

    @property
    def entries(self) -> int:
        """Entries per sequence once the step's tokens are appended."""
        return self.total_tokens // self.m


WORKLOADS = {
    # Tiny: batch 1, 4,096 tokens, m=1, one Full layer, 8 heads, D=128,
    # indexer 4x64, Top-64, window 128, 16 planted keys.
    "tiny": Workload("tiny", B=1, n=4096, m=1, D=128, H=8, H_I=4, dI=64, K=64, P=2048,
                     window=128, mode="full", planted=16),
    # Decoder decode step, Full layer: batch 8, context 65,536.
    "dec_full": Workload("dec_full", B=8, n=65536, m=1, D=512, H=64, H_I=64, dI=128, K=512,
                         P=2048, window=128, mode="full"),
    # Decoder group Reindex + 3 Reuse: batch 16, context 262,144.
    "dec_group": Workload("dec_group", B=16, n=262144, m=1, D=512, H=64, H_I=64, dI=128, K=512,
                          P=2048, window=128, mode="group", n_reuse=3),
    # Encoder prefill chunk: 8,192 new tokens over a 131,072-token prefix, m=2,
    # Full + 5 Reuse.
    "enc_prefill": Workload("enc_prefill", B=1, n=131072, m=2, D=512, H=64, H_I=64, dI=128,
                            K=512, P=0, window=128, mode="prefill", T=8192, n_reuse=5),
    # Long-context decode: batch 4, context 1,048,576, Full -> pool -> Reindex + 3 Reuse,
    # 512 planted near-duplicates of q.
    "long": Workload("long", B=4, n=1048576, m=1, D=512, H=64, H_I=64, dI=128, K=512, P=2048,
                     window=128, mode="long", n_reuse=3, planted=512),
}


def small(name: str, **over) -> Workload:
    """A workload of the same structure with some sizes replaced."""
    return dataclasses.replace(WORKLOADS[name], **over)


def _gen(seed: int, tag: str, b: int = 0) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(zlib.crc32(f"{seed}/{tag}/{b}".encode()))
    return g


def _normal_bf16(g, *shape, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(*shape, generator=g, dtype=torch.float32)
    if std != 1.0:
        x = x * std
    return x.to(torch.bfloat16)


def w_ik(wl: Workload, seed: int = 0) -> torch.Tensor:
    """Indexer projection [D][dI] bf16 ~ N(0, 1/D)."""
    return _normal_bf16(_gen(seed, "W_IK"), wl.D, wl.dI, std=wl.D ** -0.5)


def planted_positions(wl: Workload, seed: int, b: int) -> torch.Tensor:
    """Distinct token positions outside the window, ascending."""
    if wl.planted == 0:
        return torch.zeros(0, dtype=torch.int64)
    hi = wl.n - wl.window
    perm = torch.randperm(hi, generator=_gen(seed, "planted_pos", b))[: wl.planted]
    return torch.sort(perm).values


def target(wl: Workload, seed: int, b: int) -> torch.Tensor:
    return _normal_bf16(_gen(seed, "u", b), wl.D)


def context_kv(wl: Workload, seed: int, b: int, tokens: int | None = None) -> torch.Tensor:
    """Main KV rows of tokens 0..tokens-1 of sequence b, [tokens][D] bf16."""
    tokens = wl.total_tokens if tokens is None else tokens
    kv = _normal_bf16(_gen(seed, "kv", b), tokens, wl.D)
    if wl.planted:
        pos = planted_positions(wl, seed, b)
        pos = pos[pos < tokens]
        u = target(wl, seed, b).float()
        noise = torch.randn(wl.planted, wl.D, generator=_gen(seed, "kv_planted", b))[: pos.numel()]
        kv[pos] = (u[None, :] + 0.1 * noise).to(torch.bfloat16)
    return kv


def context_gate(wl: Workload, seed: int, b: int, tokens: int | None = None) -> torch.Tensor:
    """Gate logits of tokens 0..tokens-1 (m=2 workloads), [tokens][D] bf16."""
    tokens = wl.total_tokens if tokens is None else tokens
    return _normal_bf16(_gen(seed, "gate", b), tokens, wl.D)


def window_lo(wl: Workload) -> int:
    """First token whose window row exists before the step."""
    return max(0, wl.first_new - wl.window + 1)


def window_kv(wl: Workload, seed: int, layer: int, b: int) -> torch.Tensor:
    """Window-cache KV rows of one layer for tokens window_lo .. total_tokens-1,
    [rows][D] bf16 (the rows before first_new prefill the ring; the rest are
    the step's own)."""
    rows = wl.total_tokens - window_lo(wl)
    return _normal_bf16(_gen(seed, f"swa{layer}", b), rows, wl.D)


def queries(wl: Workload, seed: int, layer: int, b: int, T_q: int = 1) -> torch.Tensor:
    """Attention query heads of one layer, [T_q][H][D] bf16."""
    q = _normal_bf16(_gen(seed, f"q{layer}", b), T_q, wl.H, wl.D)
    if wl.planted:
        u = target(wl, seed, b).float()
        noise = torch.randn(T_q, wl.H, wl.D, generator=_gen(seed, f"q{layer}_planted", b))
        q = (u[None, None, :] + 0.1 * noise).to(torch.bfloat16)
    return q


def index_queries(wl: Workload, seed: int, layer: int, b: int, T_q: int = 1):
    """Indexer query heads [T_q][H_I][dI] bf16 and weights [T_q][H_I] f32 ~ U(0,1)."""
    qi = _normal_bf16(_gen(seed, f"qi{layer}", b), T_q, wl.H_I, wl.dI)
    w = torch.rand(T_q, wl.H_I, generator=_gen(seed, f"w{layer}", b), dtype=torch.float32)
    if wl.planted:
        u = target(wl, seed, b).float()
        wu = u @ w_ik(wl, seed).float()
        noise = torch.randn(T_q, wl.H_I, wl.dI, generator=_gen(seed, f"qi{layer}_planted", b))
        qi = (wu[None, None, :] + 0.1 * noise).to(torch.bfloat16)
    return qi, w


def random_indices(n_vis: int, K: int, g: torch.Generator, n_missing: int = 0) -> torch.Tensor:
    """K distinct ascending entry ids < n_vis, the last n_missing replaced by -1."""
    k = min(K, n_vis)
    keep = max(0, k - n_missing)
    idx = torch.sort(torch.randperm(n_vis, generator=g)[:k]).values.to(torch.int32)
    out = torch.full((K,), -1, dtype=torch.int32)
    out[:keep] = idx[:keep]
    return out


def bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor (for the oracle)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")
