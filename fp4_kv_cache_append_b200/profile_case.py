"""Small, self-terminating run of one workload's step for profiler captures.

    python -m fp4_kv_cache_append_b200.profile_case [--workload dec_full] [--steps 6] [--time N]
    python -m fp4_kv_cache_append_b200.profile_case --attn-rows 256 [--steps 4]

Fills one cache copy (untimed), then enqueues `steps` eager steps and exits.
With --attn-rows, runs only gather + attention (dec_full shapes: 64 heads,
D 512, Top-512 + a 128-row window) over that many query rows of synthetic
caches (16,384 entries per sequence, values like quantised N(0, 1) rows):
from 149 rows on, the launch takes the pipelined form.
Used under ncu: the launch list (one metric, one pass) and `--set full`
captures of a single kernel (-k/-s/-c).  With --time N (never under a
profiler) it then runs N more steps with CUDA events around every call and
prints each entry point's mean time per call, and for a Full scan its FP8
MMA rate (2 x indexer heads x d_I FLOP per visible entry and query row).
"""
from __future__ import annotations

import argparse

import torch

from . import csa2 as C
from . import inputs as I
from . import runner


def attention_only(rows: int, steps: int):
    import math
    wl = I.WORKLOADS["dec_full"]
    n = 16384
    g = torch.Generator(device="cuda")
    g.manual_seed(7)
    main = C.MainCache(rows, n, wl.D, wl.dI, 1)
    main.codes.random_(0, 256, generator=g)
    main.scales.random_(0x2E, 0x33, generator=g)   # E4M3 0.44 .. 0.56
    main.n_entries.fill_(n)
    swa = C.SwaCache(rows, wl.window, wl.D)
    swa.rows.random_(0, 0x40, generator=g)
    swa.rows.bitwise_or_(torch.randint(0, 2, swa.rows.shape, generator=g, device="cuda", dtype=torch.uint8) << 7)
    q = torch.randn(rows, 1, wl.H, wl.D, generator=g, device="cuda").to(torch.bfloat16)
    q_pos = torch.full((rows, 1), n - 1, dtype=torch.int32, device="cuda")
    idx = torch.rand(rows, n, generator=g, device="cuda").argsort(dim=1)[:, :wl.K]
    idx = idx.to(torch.int32).reshape(rows, 1, wl.K).contiguous()
    out = torch.empty(rows, 1, wl.H, wl.D, dtype=torch.bfloat16, device="cuda")
    ws = C.workspace(C.csa2_attn_workspace_size(rows, 1, wl.H, wl.D, wl.K, wl.window))
    for _ in range(steps):
        C.csa2_sparse_attn_decode(main, swa, q, q_pos, idx, 1.0 / math.sqrt(wl.D), out, ws=ws)
    torch.cuda.synchronize()
    flags = C.csa2_device_status()
    print(f"profile_case attention over {rows} rows: {steps} launches done, device status {flags:#x}")
    if flags:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="dec_full", choices=sorted(I.WORKLOADS))
    ap.add_argument("--steps", type=int, default=6)
    ap.add_argument("--time", type=int, default=0, help="steps to time call by call after the untimed ones")
    ap.add_argument("--attn-rows", type=int, default=0, help="only gather + attention over this many query rows")
    args = ap.parse_args()
    if args.attn_rows:
        attention_only(args.attn_rows, args.steps)
        return
    wl = I.WORKLOADS[args.workload]
    st = runner.Step(wl, seed=0, copies=1)
    st.prefill()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        st.run(copy=0)
    torch.cuda.synchronize()
    if args.time:
        events = {}
        for _ in range(args.time):
            st.run(copy=0, events=events)
        torch.cuda.synchronize()
        for name, pairs in events.items():
            ms = sorted(s_.elapsed_time(e_) for s_, e_ in pairs)
            print(f"{name:14s} {len(pairs) // args.time} call(s) per step, {sum(ms) / len(ms):9.3f} ms per call "
                  f"(min {ms[0]:.3f})")
        scan = "index_topk" if "index_topk" in events else "index_full"
        if scan in events:
            ms = min(s_.elapsed_time(e_) for s_, e_ in events[scan])
            flop = 2.0 * wl.H_I * wl.dI * float(st.n_valid.sum().item())
            print(f"{scan}: {flop / 1e12:.2f} TFLOP of FP8 MMA per call, {flop / (ms * 1e-3) / 1e12:.1f} TFLOP/s "
                  f"at the fastest call")
    flags = C.csa2_device_status()
    print(f"profile_case {args.workload}: {args.steps} steps done, device status {flags:#x}")
    if flags:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
