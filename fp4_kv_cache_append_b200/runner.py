"""Layer sequencing of a CSA2 step through the C ABI (call order only).

DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2" and its worked
example: every layer computes its own query and window KV; a Full layer owns
the main KV, scores it and picks Top-K (the decoder's first Full layer also
builds the 2,048 x 8 pool); a Reindex layer keeps the KV and rescores the
pool with its own indexer query; a Reuse layer inherits KV and indices.
Encoder groups are Full + 5 Reuse; decoder groups are Full + 3 Reuse or
Reindex + 3 Reuse (paper sec. 4.2.1).

This module holds device buffers and the order of the calls; all of the
method's arithmetic runs in libcsa2.
"""
from __future__ import annotations

import math

import torch

from . import csa2 as C
from . import inputs as I

# layer plan per workload mode: (kind, window-cache / query layer id)
PLANS = {
    "full": [("full", 0)],
    "group": [("reindex", 0), ("reuse", 1), ("reuse", 2), ("reuse", 3)],
    "long": [("full", 0), ("reindex", 1), ("reuse", 2), ("reuse", 3), ("reuse", 4)],
    "prefill": [("full", 0)] + [("reuse", l) for l in range(1, 6)],
}
POOL_LAYER = 100   # query id of the untimed Full layer that builds a group's pool


def cap_for(wl: I.Workload) -> int:
    return (wl.entries + 127) // 128 * 128


def w_cap_for(wl: I.Workload) -> int:
    return wl.window if wl.T == 1 else wl.T + wl.window - 1


class Step:
    """Caches, inputs and buffers of one workload; `run()` enqueues one step."""

    def __init__(self, wl: I.Workload, seed: int = 0, device: str = "cuda", copies: int = 1,
                 prefill_chunk: int = 16384, fused: bool = False):
        self.wl, self.seed, self.device = wl, seed, device
        self.prefill_chunk = prefill_chunk
        self.plan = PLANS[wl.mode]
        self.cap = cap_for(wl)
        self.W_cap = w_cap_for(wl)
        self.layers = [l for _, l in self.plan]
        B, D = wl.B, wl.D
        self.T_q = wl.T
        self.rows = B * self.T_q
        self.scale = 1.0 / math.sqrt(D)
        dev = device

        # ---- caches (copies: independent replicas with the same content, to
        # rotate through so that a timed step does not hit L2)
        self.main = [C.MainCache(B, self.cap, D, wl.dI, wl.m, device=dev) for _ in range(copies)]
        self.swa = [{l: C.SwaCache(B, self.W_cap, D, window=wl.window, device=dev) for l in self.layers}
                    for _ in range(copies)]
        self.w_ik = I.w_ik(wl, seed).to(dev)

        # ---- step inputs
        kv_ctx = [I.context_kv(wl, seed, b) for b in range(B)]
        self._kv_ctx = kv_ctx
        self.kv_new = torch.stack([k[wl.first_new:] for k in kv_ctx]).to(dev)          # [B][T][D]
        self.gate_new = None
        if wl.m == 2:
            g_ctx = [I.context_gate(wl, seed, b) for b in range(B)]
            self._gate_ctx = g_ctx
            self.gate_new = torch.stack([g[wl.first_new:] for g in g_ctx]).to(dev)
        lo = I.window_lo(wl)
        self.win_rows = {l: [I.window_kv(wl, seed, l, b) for b in range(B)] for l in self.layers}
        self.kv_swa_new = {l: torch.stack([r[wl.first_new - lo:] for r in self.win_rows[l]]).to(dev)
                           for l in self.layers}
        self.q = {l: torch.stack([I.queries(wl, seed, l, b, self.T_q) for b in range(B)]).to(dev)
                  for l in self.layers}
        qi_layers = [l for k, l in self.plan if k in ("full", "reindex")]
        if wl.mode == "group":
            qi_layers = qi_layers + [POOL_LAYER]
        self.q_idx, self.w = {}, {}
        for l in qi_layers:
            pairs = [I.index_queries(wl, seed, l, b, self.T_q) for b in range(B)]
            self.q_idx[l] = torch.stack([p[0] for p in pairs]).to(dev)
            self.w[l] = torch.stack([p[1] for p in pairs]).to(dev)
        self.pos0 = torch.full((B,), wl.first_new, dtype=torch.int32, device=dev)
        self.q_pos = (wl.first_new + torch.arange(self.T_q, dtype=torch.int32)).repeat(B, 1).to(dev).contiguous()

        # ---- work buffers
        P = wl.P
        self.scores = torch.empty(self.rows, self.cap, dtype=torch.float32, device=dev)
        self.n_valid = torch.empty(self.rows, dtype=torch.int32, device=dev)
        self.idx = torch.empty(self.rows, wl.K, dtype=torch.int32, device=dev)
        self.pool = torch.empty(self.rows, max(P, 16), dtype=torch.int32, device=dev)
        self.pool_scores = torch.empty(self.rows, max(P, 16) * 8, dtype=torch.float32, device=dev)
        self.out = {l: torch.empty(B, self.T_q, wl.H, D, dtype=torch.bfloat16, device=dev) for l in self.layers}
        ws_full = C.csa2_topk_workspace_size(self.rows, self.cap, wl.K, P)
        ws_re = C.csa2_topk_workspace_size(self.rows, max(P, 16) * 8, wl.K, 0)
        ws_at = C.csa2_attn_workspace_size(B, self.T_q, wl.H, D, wl.K, wl.window)
        self.ws_topk = C.workspace(max(ws_full, ws_re), dev)
        self.ws_attn = C.workspace(ws_at, dev)
        # fused: the Full layer selects from the block maxima its scan writes
        # (csa2_index_topk, contexts up to 131,072 entries); otherwise the scan
        # writes the scores and csa2_topk selects from them.  The second is
        # the faster today (measured: the fused selection's one block per row
        # is instruction-bound), so it is the default.
        self.fused = fused and wl.mode in ("full", "prefill") and self.cap <= 131072
        ws_i = (C.csa2_index_topk_workspace_size(self.rows, self.cap, wl.dI) if self.fused
                else C.csa2_index_workspace_size(self.rows, wl.dI))
        self.ws_index = C.workspace(ws_i, dev)

    # ------------------------------------------------------------------ set-up (untimed)

    def prefill(self):
        """Fill every cache copy with the context before the step's tokens."""
        wl, B, dev = self.wl, self.wl.B, self.device
        first = wl.first_new
        main0 = self.main[0]
        for c0 in range(0, first, self.prefill_chunk):   # chunk is even: no pair straddles two calls
            c1 = min(first, c0 + self.prefill_chunk)
            kv = torch.stack([k[c0:c1] for k in self._kv_ctx]).to(dev)
            gate = torch.stack([g[c0:c1] for g in self._gate_ctx]).to(dev) if wl.m == 2 else None
            pos0 = torch.full((B,), c0, dtype=torch.int32, device=dev)
            C.csa2_append_quant(main0, kv, gate, self.w_ik, None, None, pos0, c1 - c0)
        lo = I.window_lo(wl)
        for l in self.layers:
            if first > lo:
                rows = torch.stack([r[: first - lo] for r in self.win_rows[l]]).to(dev)
                pos0 = torch.full((B,), lo, dtype=torch.int32, device=dev)
                C.csa2_append_quant(None, None, None, None, self.swa[0][l], rows, pos0, first - lo)
        for cp in range(1, len(self.main)):
            for name in ("codes", "scales", "ik", "ik_scale", "n_entries", "pending_kv", "pending_gate"):
                getattr(self.main[cp], name).copy_(getattr(main0, name))
            for l in self.layers:
                self.swa[cp][l].rows.copy_(self.swa[0][l].rows)
        if wl.mode == "group":
            self._build_pool()
        torch.cuda.synchronize()

    def _build_pool(self):
        """The group head's pool comes from an (untimed) Full scan on the same cache."""
        wl = self.wl
        m = self.main[0]
        # the step's token must be in the cache for the scan: append it first
        C.csa2_append_quant(m, self.kv_new, self.gate_new, self.w_ik, None, None, self.pos0, wl.T)
        C.csa2_index_full(m, self.q_idx[POOL_LAYER], self.w[POOL_LAYER], self.q_pos, self.scores, self.n_valid,
                          ws=self.ws_index)
        C.csa2_topk(self.scores, self.cap, wl.K, self.idx, n_valid=self.n_valid, P_out=wl.P, out_pool=self.pool,
                    ws=self.ws_topk)
        self.group_pool = self.pool.clone()
        for cp in range(1, len(self.main)):
            for name in ("codes", "scales", "ik", "ik_scale", "n_entries"):
                getattr(self.main[cp], name).copy_(getattr(m, name))

    # ------------------------------------------------------------------ the step

    def run(self, copy: int = 0, events=None, external_events: bool = False):
        """Enqueue one step on the current stream.  `events`, if given, is a
        dict of entry-point name -> list of (start, end) CUDA event pairs to
        record around each call (external_events: record nodes inside a CUDA
        graph capture)."""
        wl = self.wl
        main, swa = self.main[copy], self.swa[copy]

        def timed(name, fn):
            if events is None:
                fn()
                return
            s = torch.cuda.Event(enable_timing=True, external=external_events)
            e = torch.cuda.Event(enable_timing=True, external=external_events)
            s.record()
            fn()
            e.record()
            events.setdefault(name, []).append((s, e))

        for kind, l in self.plan:
            if kind == "full":
                # the append launch also prepares the scan's indexer query
                timed("append", lambda: C.csa2_append_quant_ex(main, self.kv_new, self.gate_new, self.w_ik, swa[l],
                                                               self.kv_swa_new[l], self.pos0, wl.T, self.q_idx[l],
                                                               self.w[l], self.ws_index))
                if self.fused:
                    timed("index_topk", lambda: C.csa2_index_topk(main, None, None, self.q_pos, self.scores, wl.K,
                                                                  self.idx, n_valid=self.n_valid, P_out=wl.P,
                                                                  out_pool=self.pool if wl.P else None,
                                                                  ws=self.ws_index))
                else:
                    timed("index_full", lambda: C.csa2_index_full_prepared(main, self.q_pos, self.scores,
                                                                           self.n_valid, ws=self.ws_index))
                    timed("topk", lambda: C.csa2_topk(self.scores, self.cap, wl.K, self.idx, n_valid=self.n_valid,
                                                      P_out=wl.P, out_pool=self.pool if wl.P else None,
                                                      ws=self.ws_topk))
            elif kind == "reindex":
                timed("append", lambda: C.csa2_append_quant(None, None, None, None, swa[l], self.kv_swa_new[l],
                                                            self.pos0, wl.T))
                pool = self.group_pool if wl.mode == "group" else self.pool
                timed("index_reindex", lambda: C.csa2_index_reindex(main, self.q_idx[l], self.w[l], self.q_pos,
                                                                    pool, self.pool_scores, ws=self.ws_index))
                timed("topk", lambda: C.csa2_topk(self.pool_scores, wl.P * 8, wl.K, self.idx, pool_blocks=pool,
                                                  ws=self.ws_topk))
            else:  # reuse: own window rows and query, inherited KV and indices
                timed("append", lambda: C.csa2_append_quant(None, None, None, None, swa[l], self.kv_swa_new[l],
                                                            self.pos0, wl.T))
            timed("attn", lambda: C.csa2_sparse_attn_decode(main, swa[l], self.q[l], self.q_pos, self.idx,
                                                            self.scale, self.out[l], ws=self.ws_attn))

    # ------------------------------------------------------------------ accounting

    def launches_per_step(self) -> int:
        """libcsa2 kernel launches one step enqueues (append 1, which also
        prepares a Full scan's query; Full scan with the fused selection 2, or
        scan 1 + Top-K; Reindex 2 = query prep + scan; Top-K 1 for rows of up
        to 65,536 columns else 4 (1 for >= 128 rows of up to 131,072 without
        a pool); attention 1)."""
        wl = self.wl
        topk = lambda n_cols: 1 if n_cols <= 65536 or (self.rows >= 128 and n_cols <= 131072 and not wl.P) else 4
        n = 0
        for kind, _ in self.plan:
            n += 1 + 1   # append, attention
            if kind == "full":
                n += 2 if self.fused else 1 + topk(self.cap)
            elif kind == "reindex":
                n += 2 + topk(wl.P * 8)
        return n

    def algorithmic_bytes(self) -> dict:
        """Bytes each entry point must move per step (cold caches)."""
        wl, B, D = self.wl, self.wl.B, self.wl.D
        entry = D // 2 + D // 16
        ik = wl.dI + 4
        out = {}
        n_vis = wl.entries
        for kind, l in self.plan:
            if kind == "full":
                out["index_full"] = out.get("index_full", 0) + B * self.T_q * 0 + B * n_vis * ik \
                    + B * self.T_q * wl.H_I * (2 * wl.dI + 4)
            if kind == "reindex":
                out["index_reindex"] = out.get("index_reindex", 0) + self.rows * wl.P * 8 * ik
            att = self.rows * (wl.K * entry + wl.window * D + 2 * 2 * wl.H * D)
            out["attn"] = out.get("attn", 0) + att
            # append: new kv rows (+ gate), the entries' FP4 bytes and keys, window rows in and out
            new_entries = B * wl.T // wl.m if kind == "full" else 0
            app = B * wl.T * D * 2 * (1 if kind != "full" else (2 if wl.m == 1 else 3)) + B * wl.T * D \
                + new_entries * (entry + ik) + (D * wl.dI * 2 if kind == "full" else 0)
            out["append"] = out.get("append", 0) + app
            if kind in ("full", "reindex"):
                cols = self.cap if kind == "full" else wl.P * 8
                out["topk"] = out.get("topk", 0) + self.rows * (cols * 4 + wl.K * 4) \
                    + (self.rows * wl.P * 4 if kind == "full" and wl.P else 0)
        if self.fused:   # the scan's bytes plus the selection's: block maxima out and in, the candidates' scores
            nb = (wl.entries + 7) // 8
            out["index_topk"] = out.pop("index_full") + self.rows * (2 * nb * 4 + 8 * wl.K * 4 + wl.K * 4 + wl.P * 4)
            out.pop("topk")
        return out

    def algorithmic_flops(self) -> dict:
        """FLOPs of the contractions per step: FP8 indexer q.k over the visible
        entries (or pool columns) x heads x d_I x 2; attention S and P.V over
        K + window keys x heads x D x 4 per layer."""
        wl = self.wl
        out = {}
        for kind, _ in self.plan:
            if kind == "full":
                vis = sum(min(wl.entries, (wl.first_new + j + 1) // wl.m) for j in range(self.T_q))
                out["index_topk" if self.fused else "index_full"] = wl.B * vis * wl.H_I * wl.dI * 2
            if kind == "reindex":
                out["index_reindex"] = self.rows * wl.P * 8 * wl.H_I * wl.dI * 2
            out["attn"] = out.get("attn", 0) + self.rows * (wl.K + wl.window) * wl.H * wl.D * 4
        return out
