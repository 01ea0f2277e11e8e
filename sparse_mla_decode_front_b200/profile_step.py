"""Run a few block steps of a synthetic workload and exit (for profilers).

    python -m sparse_mla_decode_front_b200.profile_step --workload gather128 --steps 2 [--separate]
    python -m sparse_mla_decode_front_b200.profile_step --router router_ds128 --steps 3
    python -m sparse_mla_decode_front_b200.profile_step --tp-world 1 --steps 3

Uploads the workload once, runs ``--steps`` calls of the block on cuda:0 (with
``--separate``: the two calls of the separate path, qkv then attention, per step;
with ``--router CASE``: the fused RMSNorm + router top-K on that router case instead;
with ``--tp-world W``: the head split's fused o-projection + reduction on the block's
o-projection shape, every one of W ranks on this GPU),
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
    ap.add_argument("--router", default=None, choices=[c.name for c in synth.ROUTER_CASES],
                    help="run the router case instead of the block")
    ap.add_argument("--tp-world", type=int, default=0, help="run the head split's o-projection for W ranks")
    args = ap.parse_args(argv)
    if args.router:
        return _router(args)
    if args.tp_world:
        return _tp_o_proj(args)
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


def _router(args) -> int:
    import numpy as np
    from . import api
    case = synth.ROUTER_CASE_BY_NAME[args.router]
    inp = synth.make_router_inputs(case.index)
    dev = torch.device("cuda:0")
    t16 = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    x, g, w = (t16(inp[k]) for k in ("hidden_states", "gamma", "router_weights"))
    b = None if inp["router_bias"] is None else t16(inp["router_bias"])
    T, H, E, K = case.n_tokens, case.hidden, case.n_experts, case.top_k
    norm = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    aff = torch.empty((T, E), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(api.mla_router_workspace_bytes(T, H, E, K), dtype=torch.uint8, device=dev)
    for _ in range(args.steps):
        api.mla_rmsnorm_router_topk(x, g, w, b, inp["eps"], K, case.act, norm, idx, aff, ws)
    torch.cuda.synchronize()
    status = int(ws[:4].view(torch.int32).item())
    print(f"{case.name}: {args.steps} calls, {api.mla_router_launches(T, H, E, K)} kernels per call, "
          f"device status {status:#x}")
    return 0 if status == 0 else 1


def _tp_o_proj(args) -> int:
    from . import api, tp
    from .device import _to_torch
    dev = torch.device("cuda:0")
    T, K, H = 128, 16384, 7168
    x = synth.make_o_proj_inputs(T, K, H, seed=7200)
    o, w = _to_torch(x["o"], True).to(dev), _to_torch(x["o_proj_w"], True).to(dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    pb = tp.PeerBuffers.local(args.tp_world, T, H, device=dev)
    for e in range(1, args.steps + 1):
        api.mla_tp_o_proj_allreduce(o, w, pb.table(0, e), args.tp_world, ws, None)
    torch.cuda.synchronize()
    status = int(ws[:4].view(torch.int32).item())
    print(f"head-split o-projection, world {args.tp_world}: {args.steps} calls, device status {status:#x}")
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
