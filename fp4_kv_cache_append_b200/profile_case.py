"""Small, self-terminating run of one workload's step for profiler captures.

    python -m fp4_kv_cache_append_b200.profile_case [--workload dec_full] [--steps 6] [--time N]

Fills one cache copy (untimed), then enqueues `steps` eager steps and exits.
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


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="dec_full", choices=sorted(I.WORKLOADS))
    ap.add_argument("--steps", type=int, default=6)
    ap.add_argument("--time", type=int, default=0, help="steps to time call by call after the untimed ones")
    args = ap.parse_args()
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
