#!/usr/bin/env python
"""Benchmark of the CSA2 decode step over an FP4 KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one GPU): the decoder decode step of a Full layer -- batch 8,
context 65,536 tokens (m = 1), 64 query heads sharing one KV of dim 512
(FP4 E2M1 + E4M3 per 16 channels), indexer 64 heads x 128 (FP8), Top-512 plus
the 2048-block x 8 candidate pool, 128-token FP8 window.  A step is one token
for all 8 sequences: append + quantise, Full indexer scan, Top-K + pool,
sparse MQA attention (four C-ABI calls, six kernels).

Timing: W warm-up replays, then K steps as CUDA-graph replays (each graph is
one rotation over 4 independent cache copies, 280 MB of indexer keys in all,
more than the 126 MB L2, so no step finds its cache in L2), bracketed by a
barrier and a device synchronisation, the maximum over ranks.  With N > 1
(torchrun) every rank runs its own batch of 8 sequences: weak scaling, no
data-path collective.  Prints one JSON line on rank 0.

--impl reference times the CPU oracle (oracle/) on this machine's host cores
on a bounded sample of the same workload: one sequence's append, Full scores
over a slice of its entries, Top-K and pool over that slice and attention,
extrapolated to the whole step (oracle_sample).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode steps/s and achieved HBM GB/s (% of roofline) at 1 B200"
WORKLOAD = "dec_full"
WORKLOAD_DESC = ("decoder decode step, Full layer: batch 8, context 65,536, m=1, 64 heads sharing one KV of "
                 "dim 512 (FP4 E2M1 + E4M3/16ch), indexer 64x128 FP8, Top-512 + 2048x8 pool, window 128 FP8")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=24000)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--copies", type=int, default=4)
    ap.add_argument("--graph-rotations", type=int, default=8, help="cache rotations captured per graph")
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--attn-sweep", action="store_true",
                    help="print only the gather + attention batch sweep (rank 0, one GPU) and exit")
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def bf16_peak() -> float:
    """Dense bf16 tensor TFLOP/s (burst) of MEASURED_PEAKS.json, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"])
    return FALLBACK_BF16_TFLOPS


INDEX_SOURCES = ("index.cu", "common.cuh", "kernels.h")   # what builds the index kernels


def source_sha(names=INDEX_SOURCES) -> str:
    """Hash of the sources a kernel is built from (first 16 hex digits)."""
    import hashlib
    src = os.path.join(ROOT, "fp4_kv_cache_append_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(names):
        with open(os.path.join(src, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_tag: str):
    """Per-launch DRAM bytes of a kernel from a committed ncu summary, if the
    summary was taken on the current kernel source (else None)."""
    summ = os.path.join(ROOT, "profiles", f"{kernel_tag}.md")
    if not os.path.exists(summ):
        return None
    want = source_sha()
    sha = traffic = None
    with open(summ) as f:
        for line in f:
            if line.startswith("source_sha:"):
                sha = line.split(":", 1)[1].strip()
            if line.startswith("traffic_bytes_per_launch:"):
                traffic = float(line.split(":", 1)[1].strip())
    return traffic if sha == want else None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[2], float(parts[3]), parts[4:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        loaded = [r for r in rows if r[3] >= 50] or rows
        names = ["active_mask", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in loaded:
            for n, v in zip(names[1:], r[4][1:]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in loaded),
                "reasons": sorted(reasons), "samples": len(loaded)}


# --------------------------------------------------------------------------- multi-rank plumbing


def rank_seed(rank: int) -> int:
    """Each rank decodes its own batch of sequences (weak scaling)."""
    return rank


def max_over_ranks(ms: float, dist, device) -> float:
    """The job's time is the slowest rank's (device-timed) region."""
    if dist is None:
        return ms
    import torch
    tt = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(tt, op=dist.ReduceOp.MAX)
    return float(tt.item())


def job_throughput(world: int, steps: int, ms: float) -> float:
    """Steps of all ranks per second of the slowest rank."""
    return world * steps / (ms / 1e3)


# --------------------------------------------------------------------------- our arm


def run_ours(args, rank, world, dist):
    import torch

    from fp4_kv_cache_append_b200 import csa2 as C
    from fp4_kv_cache_append_b200 import inputs as I
    from fp4_kv_cache_append_b200 import runner

    C.lib()   # fails loudly without the CUDA library
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = I.WORKLOADS[WORKLOAD]
    st = runner.Step(wl, seed=rank_seed(rank), copies=args.copies)
    st.prefill()

    # eager warm-up: initialises per-device state and every kernel
    for i in range(args.copies):
        st.run(copy=i)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0

    # ---- graphs of `rot` rotations over the cache copies: the headline graph
    # has nothing between the calls (consecutive kernels overlap their launch
    # with the previous kernel's tail); the breakdown graph records events
    # around every call for the per-kernel durations and the roofline.
    rot = max(1, args.graph_rotations)
    steps_per_graph = rot * args.copies
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        st.run(copy=0)   # one more eager call on the capture stream
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for r in range(rot):
            for cp in range(args.copies):
                st.run(copy=cp)
    events = {}
    g_ev = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_ev):
        for r in range(rot):
            for cp in range(args.copies):
                st.run(copy=cp, events=events, external_events=True)
    n_graph = max(1, round(args.steps / steps_per_graph))
    K = n_graph * steps_per_graph
    for _ in range(max(3, args.warmup)):
        g.replay()
        g_ev.replay()
    torch.cuda.synchronize()

    gpu_id = None
    try:
        gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid) if rank == 0 else None
    except Exception:
        gpu_id = str(dev.index)
    if gpu_id is not None and gpu_id.startswith("GPU-GPU-"):
        gpu_id = gpu_id[4:]

    def barrier():
        if dist is not None:
            dist.barrier()

    # ---- timed region (headline)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_id) if rank == 0 else None
    if sampler:
        sampler.__enter__()
    barrier()
    torch.cuda.synchronize()
    t0.record()
    for _ in range(n_graph):
        g.replay()
    t1.record()
    torch.cuda.synchronize()
    barrier()
    if sampler:
        sampler.__exit__()
    ms = max_over_ranks(t0.elapsed_time(t1), dist, dev)
    assert C.csa2_device_status() == 0, "device status flagged during the timed region"

    # ---- timed region (breakdown): same steps with events around every call;
    # per-entry-point durations are the event pairs of its last replay
    n_ev = max(1, n_graph // 4)
    barrier()
    torch.cuda.synchronize()
    t2, t3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t2.record()
    for _ in range(n_ev):
        g_ev.replay()
    t3.record()
    torch.cuda.synchronize()
    barrier()
    ms_ev = t2.elapsed_time(t3) / (n_ev * steps_per_graph)
    kern_us = {k: statistics.mean(s.elapsed_time(e) for s, e in v) * 1e3 for k, v in events.items()}
    calls_per_step = {k: len(v) / steps_per_graph for k, v in events.items()}

    # ---- timed region (dominant kernel): the Full scan alone, back to back over
    # the rotating cache copies (cold), its query prepared by the step's append
    g_dom = torch.cuda.CUDAGraph()
    scan = lambda cp: C.csa2_index_full_prepared(st.main[cp], st.q_pos, st.scores, st.n_valid, ws=st.ws_index)
    with torch.cuda.graph(g_dom):
        for r in range(rot):
            for cp in range(args.copies):
                scan(cp)
    for _ in range(3):
        g_dom.replay()
    n_dom = max(4, n_graph // 8)
    barrier()
    torch.cuda.synchronize()
    t4, t5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t4.record()
    for _ in range(n_dom):
        g_dom.replay()
    t5.record()
    torch.cuda.synchronize()
    barrier()
    dom_us = t4.elapsed_time(t5) * 1e3 / (n_dom * steps_per_graph)
    assert C.csa2_device_status() == 0

    # ---- end to end through the public API: pinned host inputs in, result out, every step
    e2e = run_e2e(st, args.e2e_steps)

    if rank != 0:
        return None
    steps_per_s = job_throughput(world, K, ms)
    B, n = wl.B, wl.entries
    alg = st.algorithmic_bytes()
    step_bytes = sum(alg.values()) + B * (wl.D + wl.D) * 2 + B * (wl.D // 2 + wl.D // 16 + wl.dI + 4)
    idx_bytes = B * n * (wl.dI + 4)                        # 132 B per visible entry
    hbm, hbm_kind = peaks()
    # dominant kernel = the one that moves the step's bytes (the Full scan:
    # 132 B per visible entry, ~96% of the step's algorithmic bytes)
    dom = "index_full"
    dom_bytes = idx_bytes
    achieved = dom_bytes / (dom_us * 1e-6) / 1e9
    traffic = ncu_traffic(f"index_full_{WORKLOAD}")
    launches_per_step = st.launches_per_step()
    clocks = sampler.summary() if sampler else None
    return {
        "metric": METRIC, "value": steps_per_s, "unit": "steps/s", "n_gpus": world, "steps": K,
        "warmup": max(3, args.warmup), "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3/e2m1 storage, fp8+fp16 mma, f32 acc", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD}: {WORKLOAD_DESC}", "global_batch": B * world, "seq_len": wl.n,
                   "parallelism": f"dp{world} (independent batches, no collective)",
                   "l2": f"inputs larger than L2: {args.copies} rotating cache copies",
                   "timing": f"CUDA-graph replays of {steps_per_graph} steps"},
        "tokens_per_s": steps_per_s * B,
        "step_bytes": step_bytes, "step_gbs": step_bytes * steps_per_s / world / 1e9,
        "step_frac_hbm": step_bytes * steps_per_s / world / 1e9 / hbm,
        "kernels_us": {k: round(v, 3) for k, v in kern_us.items()},
        "ms_per_step_with_events": ms_ev,
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm,
                     "peak_kind": hbm_kind, "unit": "GB/s", "frac": achieved / hbm if achieved else None,
                     "traffic": traffic, "bytes_per_launch": dom_bytes, "launch_us": dom_us,
                     "per_unit": "132 B per visible entry (128 B E4M3 key + 4 B scale)",
                     "timing": "prepared Full scans back to back in a CUDA graph over 4 rotating cache copies"},
        "clocks": clocks, "e2e": e2e, "gpu_launches": launches_per_step * K,
    }


SWEEP_ROWS = (8, 16, 32, 64, 128)


def attn_batch_sweep(hbm, bf16_peak):
    """Gather + attention alone (csa2_sparse_attn_decode, dec_full shapes:
    64 heads, D 512, Top-512 + a 128-row window) at 8 ... 128 query rows.
    Each launch is timed on its own with CUDA events, after a 256 MB write
    that evicts the previous launch's lines from L2 (cold gathers).  Caches
    hold 16,384 random entries per sequence (the kernel reads only the 512
    selected rows and the window, so the context length does not enter);
    codes are random bytes, scales E4M3 in [2^-6, 2^1], window rows positive
    E4M3, q ~ N(0, 1).  Algorithmic bytes per row: 512 x 288 B gathered +
    128 x 512 B window + 64 KB q + 64 KB out = 344,064 B; FLOPs per row:
    640 keys x 64 heads x 512 x 4 = 83.9 M (S and P.V)."""
    import math

    import torch

    from fp4_kv_cache_append_b200 import csa2 as C
    from fp4_kv_cache_append_b200 import inputs as I
    wl = I.WORKLOADS[WORKLOAD]
    n = 16384
    per_row_bytes = wl.K * (wl.D // 2 + wl.D // 16) + wl.window * wl.D + 2 * wl.H * wl.D * 2
    per_row_flops = (wl.K + wl.window) * wl.H * wl.D * 4
    g = torch.Generator(device="cuda")
    g.manual_seed(20261202)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    res = []
    for rows in SWEEP_ROWS:
        main = C.MainCache(rows, n, wl.D, wl.dI, 1)
        main.codes.random_(0, 256, generator=g)
        main.scales.random_(0x28, 0x49, generator=g)
        main.n_entries.fill_(n)
        swa = C.SwaCache(rows, wl.window, wl.D)
        swa.rows.random_(0, 0x7F, generator=g)
        q = torch.randn(rows, 1, wl.H, wl.D, generator=g, device="cuda").to(torch.bfloat16)
        q_pos = torch.full((rows, 1), n - 1, dtype=torch.int32, device="cuda")
        idx = torch.rand(rows, n, generator=g, device="cuda").argsort(dim=1)[:, :wl.K]
        idx = idx.to(torch.int32).reshape(rows, 1, wl.K).contiguous()
        out = torch.empty(rows, 1, wl.H, wl.D, dtype=torch.bfloat16, device="cuda")
        ws = C.workspace(C.csa2_attn_workspace_size(rows, 1, wl.H, wl.D, wl.K, wl.window))
        call = lambda: C.csa2_sparse_attn_decode(main, swa, q, q_pos, idx, 1.0 / math.sqrt(wl.D), out, ws=ws)
        call()
        torch.cuda.synchronize()
        times = []
        for it in range(24):
            flush.fill_(it & 255)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            call()
            e1.record()
            times.append((e0, e1))
        torch.cuda.synchronize()
        us = sorted(a.elapsed_time(b) * 1e3 for a, b in times[4:])
        us = us[len(us) // 2]
        gbs = rows * per_row_bytes / us / 1e3
        tflops = rows * per_row_flops / us / 1e6
        res.append({"rows": rows, "us": round(us, 2), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                    "tflops": round(tflops, 1), "frac_bf16": round(tflops / bf16_peak, 4)})
        assert C.csa2_device_status() == 0
        del main, swa, q, idx, out, ws
    return {"per_row_bytes": per_row_bytes, "per_row_flops": per_row_flops, "timing": "median of 20 cold launches",
            "points": res}


def run_e2e(st, n_steps):
    """The same step through the public API with pinned host inputs: every
    step copies its inputs host->device and reads the attention output back,
    then synchronises.  The step's inputs live back to back (16-byte aligned)
    in one pinned host buffer and one device buffer, so a step's H2D transfer
    is a single copy; the API calls read the device buffer through views."""
    import torch

    slots = [("kv_new", None), ("kv_swa_new", 0), ("q", 0), ("q_idx", 0), ("w", 0), ("pos0", None), ("q_pos", None)]
    tensors = [getattr(st, n) if i is None else getattr(st, n)[i] for n, i in slots]
    offs, total = [], 0
    for t in tensors:
        offs.append(total)
        total += (t.numel() * t.element_size() + 15) // 16 * 16
    dev_stage = torch.empty(total, dtype=torch.uint8, device=tensors[0].device)
    host_stage = torch.empty(total, dtype=torch.uint8).pin_memory()
    for (n, i), t, o in zip(slots, tensors, offs):
        nb = t.numel() * t.element_size()
        view = dev_stage[o:o + nb].view(t.dtype).view(t.shape)
        view.copy_(t)
        host_stage[o:o + nb].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
        if i is None:
            setattr(st, n, view)
        else:
            getattr(st, n)[i] = view
    out_host = torch.empty(st.out[0].shape, dtype=st.out[0].dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in tensors)
    d2h = out_host.numel() * out_host.element_size()
    for i in range(3):
        st.run(copy=i % len(st.main))
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    for i in range(n_steps):
        dev_stage.copy_(host_stage, non_blocking=True)
        st.run(copy=i % len(st.main))
        out_host.copy_(st.out[0], non_blocking=True)
        torch.cuda.current_stream().synchronize()
    dt = time.perf_counter() - t0
    return {"value": n_steps / dt, "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n_steps, "note": "eager calls through fp4_kv_cache_append_b200.csa2, one packed H2D copy of "
                                      "the step's inputs and one D2H copy of its output, synchronised per step"}


# --------------------------------------------------------------------------- oracle (CPU) legs


def oracle_sample(seconds: float, steps: int | None = None, warmup: int = 0):
    """The oracle on a bounded sample of the workload: sequence 0's step
    (append of its token, Full scores over a contiguous slice of E of its n
    entries, Top-K and pool over that slice, attention over K + 128 keys), run
    by `threads` threads at once.  Throughput is extrapolated linearly in the
    scanned slice to n entries and to the 8 sequences of a step."""
    import concurrent.futures as cf

    import numpy as np

    import oracle
    from fp4_kv_cache_append_b200 import inputs as I

    wl = I.WORKLOADS[WORKLOAD]
    threads = min(wl.B, len(os.sched_getaffinity(0)))
    n = wl.entries
    cap = n
    om = oracle.MainCache(1, cap, wl.D, wl.dI, 1)
    kv = I.bits(I.context_kv(wl, 0, 0))
    W = I.bits(I.w_ik(wl, 0))
    first = wl.first_new
    # untimed: fill the oracle cache (threads over disjoint token ranges)
    parts = np.array_split(np.arange(first), threads)

    def fill(rg):
        if rg.size == 0:
            return
        sub = oracle.MainCache(1, cap, wl.D, wl.dI, 1)
        sub.codes, sub.scales, sub.ik, sub.ik_scale = om.codes, om.scales, om.ik, om.ik_scale
        oracle.append(sub, kv[None, rg[0]:rg[-1] + 1], None, W, None, None, np.array([rg[0]], np.int32), rg.size)

    with cf.ThreadPoolExecutor(threads) as ex:
        list(ex.map(fill, parts))
    om.n_entries[0] = first
    osw = oracle.SwaCache(1, wl.window, wl.D, window=wl.window)
    rows = I.bits(I.window_kv(wl, 0, 0, 0))
    lo = I.window_lo(wl)
    oracle.append(None, None, None, None, osw, rows[None, : first - lo], np.array([lo], np.int32), first - lo)
    qi, w = I.index_queries(wl, 0, 0, 0)
    q = I.bits(I.queries(wl, 0, 0, 0)[0])
    qi = I.bits(qi[0])
    w = w[0].numpy()
    kv_new = kv[None, first:first + 1]
    rows_new = rows[None, first - lo:]

    def one(E):
        oracle.append(om, kv_new, None, W, osw, rows_new, np.array([first], np.int32), 1)
        sc = oracle.index_scores(om, 0, qi, w, E)
        top = oracle.topk(sc, wl.K)
        oracle.block_pool(sc, wl.P)
        oracle.attention(om, osw, 0, q, top, first, 1.0 / wl.D ** 0.5)

    # calibrate the slice so that one round of `threads` samples takes the budget
    t = time.perf_counter()
    one(4096)
    t_small = time.perf_counter() - t
    per_entry = max(t_small / 4096, 1e-9)
    n_rounds = max(1, steps or 1)
    E = int(min(n, max(4096, seconds / n_rounds / per_entry)))
    for _ in range(warmup):
        with cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda _: one(E), range(threads)))
    t = time.perf_counter()
    for _ in range(n_rounds):
        with cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda _: one(E), range(threads)))
    dt = (time.perf_counter() - t) / n_rounds       # one round: `threads` sequence-samples
    seq_step_s = dt * (n / E)                         # one sequence, full scan (linear in the slice)
    step_s = seq_step_s * wl.B / threads              # 8 sequences on `threads` cores
    sample = (f"sequence 0 of {wl.B}: append 1 token + oracle scores over {E} of {n} entries + Top-{wl.K} + "
              f"pool + attention; {threads} concurrent copies per round, {n_rounds} round(s); "
              f"scaled by {n}/{E} and {wl.B}/{threads}")
    return {"value": 1.0 / step_s, "unit": "steps/s", "cores": threads, "kind": "oracle", "sample": sample}


def run_reference(args):
    t0 = time.perf_counter()
    # a few rounds of bounded samples, about a minute of oracle work in all
    cb = oracle_sample(seconds=60.0, steps=min(max(args.steps, 1), 4), warmup=min(args.warmup, 1))
    wall = time.perf_counter() - t0
    return {
        "impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / cb["value"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (int64 FP8 dots)", "data": "synthetic",
        "config": {"workload": f"{WORKLOAD}: {WORKLOAD_DESC}", "global_batch": 8, "seq_len": 65536,
                   "parallelism": "host cores (oracle)"},
        "cpu_baseline": cb, "e2e": {"value": cb["value"], "unit": "steps/s", "h2d_bytes_per_step": 0,
                                    "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }


# --------------------------------------------------------------------------- main


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as tdist
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local))
        dist = tdist
    if args.attn_sweep:
        if rank == 0:
            hbm, _ = peaks()
            print(json.dumps({"attn_batch_sweep": attn_batch_sweep(hbm, bf16_peak())}), flush=True)
        return
    try:
        res = run_ours(args, rank, world, dist)
        if rank == 0:
            res["attn_batch_sweep"] = attn_batch_sweep(peaks()[0], bf16_peak())
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = oracle_sample(seconds=args.cpu_seconds)
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
