"""Small, self-terminating run of one workload's step for profiler captures.

    python -m fp4_kv_cache_append_b200.profile_case [--workload dec_full] [--steps 6]

Fills one cache copy (untimed), then enqueues `steps` eager steps and exits.
Used under ncu: the launch list (one metric, one pass) and `--set full`
captures of a single kernel (-k/-s/-c).  Prints the number of kernel launches
of the set-up phase so captures can skip it.
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
    args = ap.parse_args()
    wl = I.WORKLOADS[args.workload]
    st = runner.Step(wl, seed=0, copies=1)
    st.prefill()
    torch.cuda.synchronize()
    for _ in range(args.steps):
        st.run(copy=0)
    torch.cuda.synchronize()
    flags = C.csa2_device_status()
    print(f"profile_case {args.workload}: {args.steps} steps done, device status {flags:#x}")
    if flags:
        raise SystemExit(1)


if __name__ == "__main__":
    main()
