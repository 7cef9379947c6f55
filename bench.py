#!/usr/bin/env python
"""Benchmark of the CSA2 decode step over an FP4 KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline workload (one GPU): the decoder decode step of a Full layer -- batch
8, context 65,536 tokens (m = 1), 64 query heads sharing one KV of dim 512
(FP4 E2M1 + E4M3 per 16 channels), indexer 64 heads x 128 (FP8), Top-512 plus
the 2048-block x 8 candidate pool, 128-token FP8 window.  A step is one token
for all 8 sequences: append + quantise, Full indexer scan, Top-K + pool,
sparse MQA attention (four C-ABI calls, four kernels).

Timing: W warm-up replays, then repeats of exactly K steps (CUDA-graph
replays rotating over 4 independent cache copies, 4 x 72 MB of step bytes,
more than the 126 MB L2, so no step finds its cache in L2), each repeat
bracketed by a barrier and a device synchronisation and timed with CUDA
events; repeats continue until they span --min-ms (at least 5); the median
repeat, maximum over ranks, is the headline.  With N > 1 (torchrun) every rank
runs its own batch of 8 sequences: weak scaling, no data-path collective.
On rank 0 of a one-GPU run the other configurations (dec_group, long,
enc_prefill) are timed the same way and reported under "configs".  Prints
one JSON line on rank 0.

--impl reference times the CPU oracle (oracle/) on this machine's host cores
on a bounded sample of the same workload: one sequence's append, Full scores
over a slice of its entries, Top-K and pool over that slice and attention,
extrapolated to the whole step (OracleSample).
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
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--copies", type=int, default=4)
    ap.add_argument("--min-ms", type=float, default=3000.0,
                    help="timed repeats of K steps continue until they span this long (at least 5 repeats)")
    ap.add_argument("--configs", default="dec_group,long,enc_prefill,ced_project",
                    help="other workloads to time on rank 0 of a one-GPU run (comma list, or 'none')")
    ap.add_argument("--e2e-steps", type=int, default=300)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=20.0)
    ap.add_argument("--attn-sweep", action="store_true",
                    help="print only the gather + attention batch sweep (rank 0, one GPU) and exit")
    a = ap.parse_args()
    a.configs = [] if a.configs in ("", "none") else [c for c in a.configs.split(",") if c]
    return a


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


KERNEL_SOURCES = {   # what builds each entry point's kernels
    "index_full": ("index.cu", "common.cuh", "kernels.h"),
    "index_topk": ("index.cu", "topk_bmax.cu", "common.cuh", "kernels.h"),
    "index_reindex": ("index.cu", "common.cuh", "kernels.h"),
    "attn": ("attn.cu", "attn_lat.cu", "common.cuh", "kernels.h"),
    "topk": ("topk_cluster.cu", "topk.cu", "common.cuh", "kernels.h"),
    "append": ("append.cu", "common.cuh", "kernels.h"),
}


def source_sha(names) -> str:
    """Hash of the sources a kernel is built from (first 16 hex digits)."""
    import hashlib
    src = os.path.join(ROOT, "fp4_kv_cache_append_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(names):
        with open(os.path.join(src, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """Per-launch DRAM bytes of an entry point's kernel from the committed ncu
    summary profiles/<kernel>_dec_full.md, if that summary was taken on the
    current kernel source (else None)."""
    summ = os.path.join(ROOT, "profiles", f"{kernel}_{WORKLOAD}.md")
    if not os.path.exists(summ) or kernel not in KERNEL_SOURCES:
        return None
    want = source_sha(KERNEL_SOURCES[kernel])
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


# --------------------------------------------------------------------------- timing helpers


def capture_steps(st, n_steps, copies, events=None):
    """A CUDA graph of exactly n_steps steps; step i uses cache copy i % copies."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n_steps):
            st.run(copy=i % copies, events=events, external_events=events is not None)
    return g


class StepGraphs:
    """Exactly K steps per replay(): K // G replays of a G-step graph and one
    replay of a (K mod G)-step graph (G a multiple of the copy count, so the
    cache rotation continues across graphs)."""

    def __init__(self, st, K, copies, max_graph=256):
        import torch
        self.K = K
        G = min(K, max(copies, max_graph // copies * copies))
        self.n_full, rem = divmod(K, G)
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            st.run(copy=0)   # one eager call on the capture stream (per-device set-up)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        self.g = capture_steps(st, G, copies) if self.n_full else None
        self.r = capture_steps(st, rem, copies) if rem else None

    def replay(self):
        for _ in range(self.n_full):
            self.g.replay()
        if self.r is not None:
            self.r.replay()


def timed_repeats(replay, min_total_ms, min_repeats, barrier):
    """Times `replay` again and again, each repeat bracketed by a barrier and a
    device synchronisation, with CUDA events on the current stream; returns
    the per-repeat milliseconds (at least min_repeats, spanning min_total_ms)."""
    import torch
    out = []
    total = 0.0
    while len(out) < min_repeats or total < min_total_ms:
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        replay()
        e1.record()
        torch.cuda.synchronize()
        barrier()
        ms = e0.elapsed_time(e1)
        out.append(ms)
        total += ms
        if len(out) > 100000:
            break
    return out


def breakdown(st, copies, n_steps, replays=3):
    """Per entry-point durations: the same steps with events around every call
    (events cut the launch overlap of consecutive kernels, so the sum is above
    the headline step time); mean over the last replay's calls."""
    import torch
    events = {}
    g = capture_steps(st, n_steps, copies, events=events)
    for _ in range(replays):
        g.replay()
    torch.cuda.synchronize()
    us = {k: statistics.mean(s.elapsed_time(e) for s, e in v) * 1e3 for k, v in events.items()}
    calls = {k: len(v) / n_steps for k, v in events.items()}
    del g
    return us, calls


def kernel_rooflines(st, kern_us, calls, hbm, fp8_peak=None):
    """Achieved GB/s (and TFLOP/s) of each entry point per call against the
    roofline: algorithmic bytes per call / its event-timed duration."""
    alg = st.algorithmic_bytes()
    flops = st.algorithmic_flops()
    out = {}
    for k, us in kern_us.items():
        n = calls.get(k, 1.0)
        if k not in alg or us <= 0:
            continue
        b = alg[k] / n
        gbs = b / (us * 1e-6) / 1e9
        d = {"us_per_call": round(us, 3), "bytes_per_call": int(b), "gbs": round(gbs, 1),
             "frac_hbm": round(gbs / hbm, 4)}
        if k in flops:
            f = flops[k] / n
            d["tflops"] = round(f / (us * 1e-6) / 1e12, 2)
            if k.startswith("index") and fp8_peak:
                d["frac_fp8_derived"] = round(d["tflops"] / fp8_peak, 4)
        out[k] = d
    return out


# --------------------------------------------------------------------------- our arm


def run_ours(args, rank, world, dist):
    import torch

    from fp4_kv_cache_append_b200 import csa2 as C
    from fp4_kv_cache_append_b200 import inputs as I
    from fp4_kv_cache_append_b200 import runner

    C.lib()   # fails loudly without the CUDA library
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = I.WORKLOADS[WORKLOAD]
    copies = args.copies
    st = runner.Step(wl, seed=rank_seed(rank), copies=copies)
    st.prefill()

    # eager warm-up: initialises per-device state and every kernel
    for i in range(copies):
        st.run(copy=i)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0

    K = max(1, args.steps)
    graphs = StepGraphs(st, K, copies)
    W = max(3, args.warmup)
    for _ in range(W):
        graphs.replay()
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

    # ---- timed region (headline): exactly K steps per repeat; repeats until
    # they span min_ms (and at least 5); the median repeat is reported
    sampler = ClockSampler(gpu_id) if rank == 0 else None
    if sampler:
        sampler.__enter__()
    reps = timed_repeats(graphs.replay, args.min_ms, 5, barrier)
    if sampler:
        sampler.__exit__()
    med = statistics.median(reps)
    ms = max_over_ranks(med, dist, dev)
    assert C.csa2_device_status() == 0, "device status flagged during the timed region"

    # ---- per-call durations (events around every call)
    steps_ev = 8 * copies
    kern_us, calls = breakdown(st, copies, steps_ev)
    ms_ev = None

    # ---- the Full scan alone, back to back over the rotating cache copies (cold)
    rot = 8
    g_dom = torch.cuda.CUDAGraph()
    scan = lambda cp: C.csa2_index_full_prepared(st.main[cp], st.q_pos, st.scores, st.n_valid, ws=st.ws_index)
    with torch.cuda.graph(g_dom):
        for r in range(rot):
            for cp in range(copies):
                scan(cp)
    for _ in range(3):
        g_dom.replay()
    dom_reps = timed_repeats(g_dom.replay, 200.0, 5, barrier)
    scan_us = statistics.median(dom_reps) * 1e3 / (rot * copies)
    del g_dom
    assert C.csa2_device_status() == 0

    # ---- end to end through the public API: pinned host inputs in, result out, every step
    e2e = run_e2e(st, args.e2e_steps)

    if rank != 0:
        return None
    steps_per_s = job_throughput(world, K, ms)
    B, n = wl.B, wl.entries
    alg = st.algorithmic_bytes()
    step_bytes = sum(alg.values())
    hbm, hbm_kind = peaks()
    fp8 = 2.0 * bf16_peak()
    kr = kernel_rooflines(st, kern_us, calls, hbm, fp8)
    scan_bytes = B * n * (wl.dI + 4) + st.rows * wl.H_I * (2 * wl.dI + 4)
    kr["scan_alone"] = {"us_per_call": round(scan_us, 3), "bytes_per_call": scan_bytes,
                        "gbs": round(scan_bytes / (scan_us * 1e-6) / 1e9, 1),
                        "frac_hbm": round(scan_bytes / (scan_us * 1e-6) / 1e9 / hbm, 4),
                        "timing": "prepared Full scans (csa2_index_full_prepared) back to back over the cache copies"}
    # the roofline object names the entry point with the largest share of the
    # step time, at its duration measured inside the step (events)
    shares = {k: kern_us[k] * calls[k] for k in kern_us}
    dom = max(shares, key=shares.get)
    dom_bytes = alg[dom] / calls[dom]
    dom_us = kern_us[dom]
    achieved = dom_bytes / (dom_us * 1e-6) / 1e9
    launches_per_step = st.launches_per_step()
    clocks = sampler.summary() if sampler else None
    return {
        "metric": METRIC, "value": steps_per_s, "unit": "steps/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3/e2m1 storage, fp8+fp16 mma, f32 acc", "data": "synthetic",
        "config": config_dict(world, copies),
        "repeats": len(reps), "timed_ms_total": sum(reps),
        "ms_per_step_spread": [min(reps) / K, max(reps) / K],
        "tokens_per_s": steps_per_s * B,
        "step_bytes": step_bytes, "step_gbs": step_bytes * steps_per_s / world / 1e9,
        "step_frac_hbm": step_bytes * steps_per_s / world / 1e9 / hbm,
        "kernels_us": {k: round(v, 3) for k, v in kern_us.items()},
        "kernel_rooflines": kr,
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": hbm,
                     "peak_kind": hbm_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": ncu_traffic(dom), "bytes_per_launch": dom_bytes, "launch_us": dom_us,
                     "share_of_step": shares[dom] / sum(shares.values()),
                     "per_unit": PER_UNIT[dom],
                     "timing": "CUDA events around each call inside the step graph"},
        "clocks": clocks, "e2e": e2e, "launches_per_step": launches_per_step,
        "gpu_launches": launches_per_step * K * len(reps),
    }


PER_UNIT = {
    "index_full": "132 B per visible entry and sequence (128 B E4M3 key + 4 B scale) + the query rows",
    "index_topk": "the scan's 132 B per visible entry + the query rows, plus the selection's block maxima "
                  "(4 B per 8 entries, written and read), the candidates' scores (8 x K x 4 B) and the outputs",
    "attn": "344,064 B per query row and layer: 512 x 288 B gathered FP4 entries + 128 x 512 B window rows "
            "+ 64 KB q + 64 KB out",
    "topk": "4 B per scored column read + 4 B per selected index / pool block written",
    "append": "the new entries' kv rows + FP4 codes/scales + indexer key + window rows + W_IK",
    "index_reindex": "132 B per pool column (P x 8 per row)",
}


def config_dict(world, copies):
    return {"workload": f"{WORKLOAD}: {WORKLOAD_DESC}", "global_batch": 8 * world, "seq_len": 65536,
            "parallelism": f"dp{world} (independent batches, no collective)",
            "l2": f"inputs larger than L2: {copies} rotating cache copies (~{copies * 72} MB of step bytes)",
            "timing": "CUDA-graph replays of exactly `steps` steps per repeat; median repeat"}


OTHER_CONFIGS = {
    # name: (cache copies rotated so a step's bytes are not L2-resident, steps per timed repeat)
    "dec_group": (3, 24),
    "long": (1, 8),
    "enc_prefill": (1, 1),
}


def run_other_configs(args, hbm, barrier):
    """The BASELINE configs other than the headline's, each timed as one
    median over repeats of whole steps (CUDA graphs), with a per-call
    breakdown and the dominant call's roofline fraction."""
    import gc

    import torch

    from fp4_kv_cache_append_b200 import csa2 as C
    from fp4_kv_cache_append_b200 import inputs as I
    from fp4_kv_cache_append_b200 import runner
    out = {}
    fp8 = 2.0 * bf16_peak()
    for name in args.configs:
        if name == "ced_project":
            out[name] = ced_project_config(hbm, barrier)
            continue
        copies, n_steps = OTHER_CONFIGS[name]
        wl = I.WORKLOADS[name]
        t0 = time.perf_counter()
        st = runner.Step(wl, seed=0, copies=copies)
        st.prefill()
        for i in range(copies):
            st.run(copy=i)
        torch.cuda.synchronize()
        assert C.csa2_device_status() == 0
        graphs = StepGraphs(st, n_steps, copies)
        for _ in range(3):
            graphs.replay()
        reps = timed_repeats(graphs.replay, 300.0, 5, barrier)
        ms = statistics.median(reps) / n_steps
        kern_us, calls = breakdown(st, copies, n_steps, replays=2)
        alg = st.algorithmic_bytes()
        flops = st.algorithmic_flops()
        kr = kernel_rooflines(st, kern_us, calls, hbm, fp8)
        shares = {k: kern_us[k] * calls[k] for k in kern_us}
        dom = max(shares, key=shares.get)
        steps_s = 1e3 / ms
        d = {"workload": WORKLOAD_DESCS[name], "ms_per_step": ms, "steps_per_s": steps_s,
             "tokens_per_s": steps_s * wl.B * wl.T, "repeats": len(reps), "steps_per_repeat": n_steps,
             "bytes_per_step": int(sum(alg.values())), "flops_per_step": int(sum(flops.values())),
             "step_gbs": sum(alg.values()) / (ms * 1e-3) / 1e9,
             "step_frac_hbm": sum(alg.values()) / (ms * 1e-3) / 1e9 / hbm,
             "kernels_us": {k: round(v, 3) for k, v in kern_us.items()}, "calls_per_step": calls,
             "kernel_rooflines": kr, "dominant": dom, "dominant_share": shares[dom] / sum(shares.values()),
             "l2": f"{copies} rotating cache copies" if copies > 1 else "a step's bytes exceed L2",
             "setup_s": round(time.perf_counter() - t0, 1)}
        if name == "enc_prefill":
            k_ix = "index_topk" if "index_topk" in kr else "index_full"
            d["index_full_fp8"] = {"call": k_ix, "tflops": kr[k_ix]["tflops"], "peak_tflops": fp8,
                                   "peak_kind": "derived: 2 x the measured dense bf16 burst (no FP8 peak is measured)",
                                   "frac": kr[k_ix]["tflops"] / fp8}
        assert C.csa2_device_status() == 0
        out[name] = d
        del graphs, st
        gc.collect()
        torch.cuda.empty_cache()
    return out


CED_SHAPE = dict(T=8192, d_model=4096, D=512, dI=128)


def ced_project_config(hbm, barrier):
    """The CED decoder-KV producer (csa2_append_project): one prefill chunk's
    decoder-layer KV kv = H W_KV (bf16 tcgen05 GEMM, FP4 E2M1/E4M3 quantised
    in its epilogue) plus the entries' FP8 indexer keys, B = 1, T = 8,192
    tokens, d_model = 4,096 (the pages give no hidden size: our choice),
    D = 512, d_I = 128.  H ~ N(0, 1), W_KV ~ N(0, 1/d_model), W_IK ~ N(0, 1/D)
    (bf16).  Three H copies (201 MB, larger than L2) rotate; a CUDA graph of
    12 calls per repeat, median over repeats."""
    import torch

    from fp4_kv_cache_append_b200 import csa2 as C
    T, dm, D, dI = (CED_SHAPE[k] for k in ("T", "d_model", "D", "dI"))
    g = torch.Generator(device="cuda")
    g.manual_seed(20261203)
    dev = "cuda"
    copies = 3
    Hs = [torch.randn(1, T, dm, generator=g, device=dev).to(torch.bfloat16) for _ in range(copies)]
    w_kv = (torch.randn(dm, D, generator=g, device=dev) / dm ** 0.5).to(torch.bfloat16)
    w_ik = (torch.randn(D, dI, generator=g, device=dev) / D ** 0.5).to(torch.bfloat16)
    main = C.MainCache(1, T, D, dI, 1, device=dev)
    pos0 = torch.zeros(1, dtype=torch.int32, device=dev)
    for cp in range(copies):
        C.csa2_append_project(main, Hs[cp], w_kv, w_ik, pos0)
    torch.cuda.synchronize()
    assert C.csa2_device_status() == 0
    n = 12
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(n):
            C.csa2_append_project(main, Hs[i % copies], w_kv, w_ik, pos0)
    for _ in range(3):
        graph.replay()
    reps = timed_repeats(graph.replay, 200.0, 5, barrier)
    ms = statistics.median(reps) / n
    gemm_flops = 2.0 * T * dm * D
    key_flops = 2.0 * T * D * dI
    nbytes = T * dm * 2 + dm * D * 2 + D * dI * 2 + T * (D // 2 + D // 16 + dI + 4)
    peak = bf16_peak()
    tflops = gemm_flops / (ms * 1e-3) / 1e12
    del graph
    assert C.csa2_device_status() == 0
    return {"workload": "CED decoder-KV producer: kv = H W_KV (bf16 GEMM, FP4-quantised in the epilogue) + FP8 "
                        f"indexer keys; B 1, T {T}, d_model {dm} (our choice: the pages give no hidden size), D {D}, "
                        f"d_I {dI}",
            "ms_per_call": ms, "tokens_per_s": T / (ms * 1e-3), "repeats": len(reps), "calls_per_repeat": n,
            "gemm_flops": gemm_flops, "key_flops": key_flops, "bytes_per_call": nbytes,
            "gemm_tflops": tflops, "peak_tflops": peak, "peak_kind": "dense bf16 burst (measured, else fallback)",
            "frac_bf16": tflops / peak, "gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm,
            "l2": f"{copies} rotating H copies ({copies * T * dm * 2 // 2**20} MiB)"}


WORKLOAD_DESCS = {
    "dec_group": "decoder group Reindex + 3 Reuse: batch 16, context 262,144, m=1, 64 heads, KV dim 512 FP4, "
                 "Reindex over the 2048 x 8 pool of an (untimed) Full scan, Top-512, window 128",
    "long": "long-context decode: batch 4, context 1,048,576, m=1, Full scan -> 2048 x 8 pool -> Reindex + 3 Reuse, "
            "64 heads, KV dim 512, Top-512, window 128, 512 planted keys",
    "enc_prefill": "encoder prefill chunk: 8,192 new tokens over a 131,072-token prefix, m=2 -> 65,536 + 4,096 "
                   "entries, Full + 5 Reuse, causal, 64 heads, KV dim 512, Top-512, window 128",
}


SWEEP_ROWS = (8, 16, 32, 64, 128, 256, 1024)   # from 256 rows the launch takes several waves (pipelined form)
SWEEP_WINDOW_ONLY_ROWS = (8, 128)   # K = 0: the SWA-only layers


def attn_batch_sweep(hbm, bf16_peak):
    """Gather + attention alone (csa2_sparse_attn_decode, dec_full shapes:
    64 heads, D 512, Top-512 + a 128-row window) at 8 ... 1,024 query rows
    (both attention forms), and the window-only form (K = 0, the SWA-only
    layers) at 8 and 128 rows.  Each launch is timed on its own with CUDA
    events, after a 256 MB write that evicts the previous launch's lines from
    L2 (cold gathers).  Caches hold 16,384 random entries per sequence (the
    kernel reads only the 512 selected rows and the window, so the context
    length does not enter); values distributed like quantised N(0, 1) rows:
    codes random bytes, scales E4M3 in [0.44, 0.56] (amax / 6 of a normal
    16-channel group), window rows E4M3 of magnitude below 2 with random
    signs, q ~ N(0, 1).  Algorithmic bytes per row: 512 x 288 B gathered +
    128 x 512 B window + 64 KB q + 64 KB out = 344,064 B; FLOPs per row:
    640 keys x 64 heads x 512 x 4 = 83.9 M (S and P.V)."""
    import math

    import torch

    from fp4_kv_cache_append_b200 import csa2 as C
    from fp4_kv_cache_append_b200 import inputs as I
    wl = I.WORKLOADS[WORKLOAD]
    n = 16384
    row_bytes = lambda K: K * (wl.D // 2 + wl.D // 16) + wl.window * wl.D + 2 * wl.H * wl.D * 2
    row_flops = lambda K: (K + wl.window) * wl.H * wl.D * 4
    g = torch.Generator(device="cuda")
    g.manual_seed(20261202)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    res = []
    for rows, K in [(r, wl.K) for r in SWEEP_ROWS] + [(r, 0) for r in SWEEP_WINDOW_ONLY_ROWS]:
        main = C.MainCache(rows, n, wl.D, wl.dI, 1)
        main.codes.random_(0, 256, generator=g)
        main.scales.random_(0x2E, 0x33, generator=g)   # E4M3 0.44 .. 0.56: amax / 6 of N(0, 1) groups
        main.n_entries.fill_(n)
        swa = C.SwaCache(rows, wl.window, wl.D)
        swa.rows.random_(0, 0x40, generator=g)          # E4M3 magnitudes below 2, random signs: N(0, 1)-like rows
        swa.rows.bitwise_or_(torch.randint(0, 2, swa.rows.shape, generator=g, device="cuda", dtype=torch.uint8) << 7)
        q = torch.randn(rows, 1, wl.H, wl.D, generator=g, device="cuda").to(torch.bfloat16)
        q_pos = torch.full((rows, 1), n - 1, dtype=torch.int32, device="cuda")
        idx = None
        if K:
            idx = torch.rand(rows, n, generator=g, device="cuda").argsort(dim=1)[:, :K]
            idx = idx.to(torch.int32).reshape(rows, 1, K).contiguous()
        out = torch.empty(rows, 1, wl.H, wl.D, dtype=torch.bfloat16, device="cuda")
        ws = C.workspace(C.csa2_attn_workspace_size(rows, 1, wl.H, wl.D, K, wl.window))
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
        gbs = rows * row_bytes(K) / us / 1e3
        tflops = rows * row_flops(K) / us / 1e6
        res.append({"rows": rows, "K": K, "us": round(us, 2), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4),
                    "tflops": round(tflops, 1), "frac_bf16": round(tflops / bf16_peak, 4)})
        assert C.csa2_device_status() == 0
        del main, swa, q, idx, out, ws
    return {"per_row_bytes": row_bytes(wl.K), "per_row_bytes_window_only": row_bytes(0),
            "per_row_flops": row_flops(wl.K), "timing": "median of 20 cold launches", "points": res}


def run_e2e(st, n_steps):
    """The same step through the public API with pinned host inputs: every
    step copies its inputs host->device and reads the attention output back
    to pinned host memory.  The step's inputs live back to back (16-byte
    aligned) in one pinned host buffer, so a step's H2D transfer is a single
    copy; the API calls read a device copy of it through views.  Steps are
    pipelined as a serving loop would run them: one CUDA graph per step
    (captured once per input stage and cache copy, then replayed) holds the
    step's calls and, on two side branches, the H2D copy of the next step's
    inputs into the other input stage and the D2H copy of the previous step's
    output, so both copies overlap the step's kernels and the host issues one
    launch per step; the host waits for step i-1's graph (and with it step
    i-2's result on the host) before it issues step i+1."""
    import torch

    slots = [("kv_new", None), ("kv_swa_new", 0), ("q", 0), ("q_idx", 0), ("w", 0), ("pos0", None), ("q_pos", None)]
    tensors = [getattr(st, n) if i is None else getattr(st, n)[i] for n, i in slots]
    offs, total = [], 0
    for t in tensors:
        offs.append(total)
        total += (t.numel() * t.element_size() + 15) // 16 * 16
    dev = tensors[0].device
    host_stage = torch.empty(total, dtype=torch.uint8).pin_memory()
    stages, views = [], []
    for _ in range(2):
        ds = torch.empty(total, dtype=torch.uint8, device=dev)
        vs = []
        for (n, i), t, o in zip(slots, tensors, offs):
            nb = t.numel() * t.element_size()
            view = ds[o:o + nb].view(t.dtype).view(t.shape)
            view.copy_(t)
            vs.append(view)
        stages.append(ds)
        views.append(vs)
    for t, o in zip(tensors, offs):
        nb = t.numel() * t.element_size()
        host_stage[o:o + nb].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
    outs = [st.out[0], torch.empty_like(st.out[0])]
    out_host = [torch.empty(st.out[0].shape, dtype=st.out[0].dtype).pin_memory() for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in tensors)
    d2h = out_host[0].numel() * out_host[0].element_size()

    def use(k):   # point the step's inputs and output at stage k
        for (n, i), v in zip(slots, views[k]):
            if i is None:
                setattr(st, n, v)
            else:
                getattr(st, n)[i] = v
        st.out[0] = outs[k]

    for i in range(3):
        use(i % 2)
        st.run(copy=i % len(st.main))
    torch.cuda.synchronize()
    # graph (k, c): step on input stage k and cache copy c, writing outs[k];
    # side branches: host -> stage 1-k (the next step's inputs) and
    # outs[1-k] -> out_host[1-k] (the previous step's result)
    ncp = len(st.main)
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    graphs = [[torch.cuda.CUDAGraph() for _ in range(ncp)] for _ in range(2)]
    for k in range(2):
        use(k)
        for c in range(ncp):
            with torch.cuda.graph(graphs[k][c]):
                cap = torch.cuda.current_stream()
                up.wait_stream(cap)
                with torch.cuda.stream(up):
                    stages[1 - k].copy_(host_stage, non_blocking=True)
                down.wait_stream(cap)
                with torch.cuda.stream(down):
                    out_host[1 - k].copy_(outs[1 - k], non_blocking=True)
                st.run(copy=c)
                cap.wait_stream(up)
                cap.wait_stream(down)
    torch.cuda.synchronize()
    comp = torch.cuda.current_stream()
    done = [torch.cuda.Event(), torch.cuda.Event()]
    t0 = time.perf_counter()
    stages[0].copy_(host_stage, non_blocking=True)   # step 0's inputs
    for i in range(n_steps):
        k = i % 2
        graphs[k][i % ncp].replay()
        done[k].record(comp)
        if i >= 1:
            done[1 - k].synchronize()   # step i-1's graph ran: step i-2's result is on the host
    k = (n_steps - 1) % 2
    out_host[k].copy_(outs[k], non_blocking=True)   # the last step's result
    comp.synchronize()
    dt = time.perf_counter() - t0
    use(0)
    return {"value": n_steps / dt, "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n_steps, "note": "the step's calls through fp4_kv_cache_append_b200.csa2 in one CUDA graph per "
                                      "step (captured once per input stage and cache copy, replayed); the graph "
                                      "also copies the next step's inputs (one packed H2D copy from pinned memory) "
                                      "and the previous step's output (one D2H copy to pinned memory) on side "
                                      "branches that overlap the kernels; the host waits for every graph, so each "
                                      "result reaches the host two steps after its own"}


# --------------------------------------------------------------------------- oracle (CPU) legs


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class OracleSample:
    """The oracle on a bounded sample of the workload: sequence 0's step
    (append of its token, Full scores over a contiguous slice of E of its n
    entries, Top-K and pool over that slice, attention over K + 128 keys).
    measure(threads, ...) runs `threads` such samples at once per round;
    throughput is extrapolated linearly in the scanned slice to n entries and
    to the 8 sequences of a step."""

    def __init__(self):
        import concurrent.futures as cf

        import numpy as np

        import oracle
        from fp4_kv_cache_append_b200 import inputs as I

        wl = self.wl = I.WORKLOADS[WORKLOAD]
        self.cores = len(os.sched_getaffinity(0))
        fill_threads = min(wl.B, self.cores)
        n = self.n = wl.entries
        om = self.om = oracle.MainCache(1, n, wl.D, wl.dI, 1)
        kv = I.bits(I.context_kv(wl, 0, 0))
        W = I.bits(I.w_ik(wl, 0))
        first = wl.first_new
        # untimed: fill the oracle cache (threads over disjoint token ranges)
        parts = np.array_split(np.arange(first), fill_threads)

        def fill(rg):
            if rg.size == 0:
                return
            sub = oracle.MainCache(1, n, wl.D, wl.dI, 1)
            sub.codes, sub.scales, sub.ik, sub.ik_scale = om.codes, om.scales, om.ik, om.ik_scale
            oracle.append(sub, kv[None, rg[0]:rg[-1] + 1], None, W, None, None, np.array([rg[0]], np.int32),
                          rg.size)

        with cf.ThreadPoolExecutor(fill_threads) as ex:
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

        self.one = one
        t = time.perf_counter()
        one(4096)
        self.per_entry = max((time.perf_counter() - t) / 4096, 1e-9)

    def measure(self, threads: int, seconds: float, rounds: int = 1, warmup: int = 0):
        import concurrent.futures as cf
        wl, n = self.wl, self.n
        E = int(min(n, max(4096, seconds / rounds / self.per_entry)))
        with cf.ThreadPoolExecutor(threads) as ex:
            for _ in range(warmup):
                list(ex.map(lambda _: self.one(E), range(threads)))
            t = time.perf_counter()
            for _ in range(rounds):
                list(ex.map(lambda _: self.one(E), range(threads)))
            dt = (time.perf_counter() - t) / rounds     # one round: `threads` sequence-samples at once
        seq_step_s = dt * (n / E)                         # one sequence, full scan (linear in the slice)
        step_s = seq_step_s * wl.B / threads              # 8 sequences on `threads` cores
        sample = (f"sequence 0 of {wl.B}: append 1 token + oracle scores over {E} of {n} entries + Top-{wl.K} + "
                  f"pool + attention; {threads} concurrent copies per round, {rounds} round(s); "
                  f"scaled by {n}/{E} and {wl.B}/{threads}")
        return {"value": 1.0 / step_s, "unit": "steps/s", "cores": threads, "kind": "oracle", "sample": sample}


def cpu_baseline(seconds: float):
    """The oracle on all host cores (up to one per sequence), and single-threaded."""
    o = OracleSample()
    mt = o.measure(min(o.wl.B, o.cores), seconds)
    one = o.measure(1, seconds / 2)
    mt.update({"value_1t": one["value"], "sample_1t": one["sample"], "cpu_model": cpu_model(),
               "host_cores": o.cores})
    return mt


def run_reference(args):
    t0 = time.perf_counter()
    o = OracleSample()
    # a few rounds of bounded samples, about a minute of oracle work in all
    threads = min(o.wl.B, o.cores)
    cb = o.measure(threads, 60.0, rounds=min(max(args.steps, 1), 4), warmup=min(args.warmup, 1))
    cb.update({"cpu_model": cpu_model(), "host_cores": o.cores})
    wall = time.perf_counter() - t0
    return {
        "impl": "reference", "metric": METRIC, "value": cb["value"], "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / cb["value"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 (int64 FP8 dots)", "data": "synthetic",
        "config": config_dict(args.gpus, args.copies),
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
            if world == 1 and args.configs:
                res["configs"] = run_other_configs(args, peaks()[0], lambda: None)
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(seconds=args.cpu_seconds)
            print(json.dumps(res), flush=True)
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
