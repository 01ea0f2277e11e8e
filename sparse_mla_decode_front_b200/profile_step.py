"""Run a few block steps of a synthetic workload and exit (for profilers).

    python -m sparse_mla_decode_front_b200.profile_step --workload gather128 --steps 2 [--separate]

Uploads the workload once, runs ``--steps`` calls of the block on cuda:0 (with
``--separate``: the two calls of the separate path, qkv then attention, per step),
synchronises and checks the device status word. Launch count per step is
printed so a profiler's skip/count options can be set (e.g. ncu -s / -c).
"""
from __future__ import annotations

import argparse
import sys

import torch

from . import synth
from .device import DecodeStep


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="gather128", choices=[w.name for w in synth.WORKLOADS])
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--separate", action="store_true", help="the separate qkv and attention calls")
    args = ap.parse_args(argv)
    step = DecodeStep(synth.make_inputs(synth.WORKLOAD_BY_NAME[args.workload].index), device="cuda:0")
    for _ in range(args.steps):
        if args.separate:
            step.run_separate()
        else:
            step.run()
    torch.cuda.synchronize()
    status = step.device_status()
    per_step = "two calls" if args.separate else f"{step.n_launches} kernels"
    print(f"{args.workload}: {args.steps} steps, {per_step} per step, device status {status:#x}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
