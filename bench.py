#!/usr/bin/env python
"""Benchmark of the sparse MLA gather-decode block step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one call of the block (index resolve, front-fold with the cache
write, gathered latent attention, out-absorption, o-projection) over one
batch of synthetic DeepSeek-V3.2-shaped decode tokens whose inputs are
already resident in HBM. Default workload: gather128 (128 tokens, 128 heads,
2048 selected keys per token over a 1M-row paged cache). L2 is flushed (a
256 MB write) before every timed step and each step is timed on the device
with CUDA events, then summed. With N > 1 (torchrun) every rank runs its own
replica batch (data parallel over sequences, no collective on the data path);
the time is the max over ranks and the value counts all ranks' tokens.

The ``e2e`` value runs back-to-back steps through the public API as a serving
loop does: every step's per-step inputs are copied from pinned host memory and
its output read back, the copies overlapped with the neighbouring steps'
compute; the serial figure (one step at a time) is reported beside it.

Prints ONE JSON line (rank 0). ``--impl reference`` times the CPU fp64
oracle instead, on a bounded sample of the same workload's tokens.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from sparse_mla_decode_front_b200 import synth  # noqa: E402

METRIC = "MLA gather-decode block us/step & tokens/s; achieved HBM GB/s vs peak"
ROW_BYTES = lambda d: 2 * d.kv_row_dim


# ---------------------------------------------------------------------------
# algorithmic bytes and flops per stage
# ---------------------------------------------------------------------------

def algorithmic(inp) -> dict:
    """Bytes that must move and flops that must run, per stage of one step.

    Bytes: every weight once, the valid gathered rows (kv_row_dim bf16 each),
    the cache-row writes, hidden in / out, and the index tensors (plus one
    block-table entry per kept key). Intermediates are not counted.
    """
    d = inp["dims"]
    T, H, Lq, L, dn, dr, dv, h, R = (d.n_tokens, d.hidden, d.q_lora_rank, d.kv_lora_rank,
                                     d.qk_nope_head_dim, d.qk_rope_head_dim, d.v_head_dim,
                                     d.n_heads, d.kv_row_dim)
    pos = inp["positions"][:, None]
    gi = inp["gather_indices"]
    n_valid = int(((gi >= 0) & (gi <= pos)).sum())
    bf, f4, i4 = 2, 4, 4
    st = {}
    st["index_resolve"] = dict(bytes=i4 * (T * d.n_prior + T + n_valid), flops=0)
    w_fold = bf * (H * Lq + H * R + Lq * h * (dn + dr) + h * dn * L)
    st["front_fold"] = dict(bytes=w_fold + bf * T * H + f4 * (H + Lq + L + T * dr) + bf * T * R + i4 * T,
                            flops=2 * T * (H * Lq + H * R + Lq * h * (dn + dr) + h * dn * L))
    st["core"] = dict(bytes=bf * R * n_valid, flops=2 * h * (R + L) * n_valid)
    st["out_absorb"] = dict(bytes=bf * h * dv * L, flops=2 * T * h * dv * L)
    st["o_proj"] = dict(bytes=bf * h * dv * H + bf * T * H, flops=2 * T * h * dv * H)
    tot = dict(bytes=sum(v["bytes"] for v in st.values()), flops=sum(v["flops"] for v in st.values()))
    return dict(stages=st, total=tot, n_valid=n_valid)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            j = json.load(fh)
        return dict(hbm_gbs=j["hbm_gbs"], bf16_tflops=j["bf16_tflops"],
                    bf16_tflops_sustained=j.get("bf16_tflops_sustained", j["bf16_tflops"]),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[i] for _, _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ---------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_tokens_per_s(inp, n_tok: int, repeats: int = 1):
    """Seconds of ``repeats`` oracle calls on a sample of ``n_tok`` tokens (every cache row is
    written, attention and output for the sample), and the sample."""
    import oracle
    d = inp["dims"]
    toks = list(np.linspace(0, d.n_tokens - 1, n_tok).round().astype(int))
    times = []
    for _ in range(repeats):
        t0 = time.perf_counter()
        oracle.block(inp, tokens=toks)       # writes every row, attends for the sample
        times.append(time.perf_counter() - t0)
    return times, toks


def cpu_baseline(inp, one_thread_tokens: int = 32) -> dict:
    """The fp64 oracle as it stands on this host: the median of 3 whole steps at all the
    cores the process may use, and the median of 3 runs on a sample of tokens at one
    thread (BLAS/OpenMP pools limited with threadpoolctl)."""
    from threadpoolctl import threadpool_limits
    d = inp["dims"]
    all_t, _ = oracle_tokens_per_s(inp, d.n_tokens, repeats=3)
    sec = statistics.median(all_t)
    n1 = max(1, min(d.n_tokens, one_thread_tokens))
    with threadpool_limits(1):
        one_t, _ = oracle_tokens_per_s(inp, n1, repeats=3)
    sec1 = statistics.median(one_t)
    return {"value": d.n_tokens / sec, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "ms_per_step": 1e3 * sec,
            "sample": f"whole step: all {d.n_tokens} tokens (every cache row written, attention and output "
                      f"for every token), median of 3 runs of {', '.join(f'{x:.2f}' for x in all_t)} s",
            "single_thread": {"value": n1 / sec1, "unit": "tokens/s", "cores": 1,
                              "sample": f"{n1} of {d.n_tokens} tokens (every cache row written, attention "
                                        f"and output for the sample), median of 3 runs of "
                                        f"{', '.join(f'{x:.2f}' for x in one_t)} s"}}


def run_reference(args, wl):
    """The reference arm: the CPU fp64 oracle as it stands, on the host cores. Each step
    is one whole block call of the workload (every token), timed; no extrapolation."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    t_run0 = time.perf_counter()
    inp = synth.make_inputs(wl.index)
    d = inp["dims"]
    for _ in range(args.warmup):
        oracle_tokens_per_s(inp, d.n_tokens)
    times = []
    for _ in range(args.steps):
        t, _ = oracle_tokens_per_s(inp, d.n_tokens)
        times += t
    sec = statistics.mean(times)
    value = d.n_tokens / sec
    cores = blas_threads()
    sample = (f"whole steps: all {d.n_tokens} tokens per step (every cache row written, attention and "
              f"output for every token); mean of {args.steps} timed steps after {args.warmup} warm-up steps")
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sec, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "n_tokens": d.n_tokens, "n_heads": d.n_heads,
                       "n_prior": d.n_prior, "hidden": d.hidden},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    wall = time.perf_counter() - t_run0
    # the timed whole steps happened inside this run: their sum cannot exceed its wall clock
    line["consistency"] = {"timed_seconds": sum(times), "run_wall_seconds": wall,
                           "fits_in_driver_run": sum(times) <= wall}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def replica_seed(workload_index: int, rank: int):
    """Seed of a rank's replica batch: rank 0 decodes the canonical workload."""
    return None if rank == 0 else 1000 + workload_index + 7919 * rank


def max_over_ranks(values, device=None):
    """Element-wise max of a list of floats over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def profiled_traffic(stage: str, workload: str):
    """DRAM bytes per launch of the stage's dominant kernel from its committed ncu summary
    (profiles/<kernel>_<workload>.md), or None when there is none or the kernel's source
    has changed since the counters were taken (the summary records the source's sha256)."""
    import hashlib
    kernels = {"core": ("core_tc", "sparse_mla_decode_front_b200/csrc/core_tc.cu")}
    if stage not in kernels:
        return None
    kern, src = kernels[stage]
    root = os.path.dirname(os.path.abspath(__file__))
    try:
        text = open(os.path.join(root, "profiles", f"{kern}_{workload}.md")).read()
        digest = hashlib.sha256(open(os.path.join(root, src), "rb").read()).hexdigest()
    except OSError:
        return None
    fields = dict(line.split(":", 1) for line in text.splitlines()
                  if line.startswith(("traffic_bytes_per_launch:", "source_sha256:")))
    if fields.get("source_sha256", "").strip() != digest:
        return None
    try:
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def gpu_uuid(dev) -> str:
    import torch
    try:
        u = torch.cuda.get_device_properties(dev).uuid
        return "GPU-" + str(u)
    except Exception:
        return str(dev.index or 0)


def time_router(dev, flush, timed_steps, args):
    """Graph-replayed fused RMSNorm + router top-K on the DeepSeek-V3 router shape
    (T=128, H=7168, E=256, K=8, sigmoid, bias); per-call ms list and the case."""
    import torch
    from sparse_mla_decode_front_b200 import api
    case = synth.ROUTER_CASE_BY_NAME["router_ds128"]
    inp = synth.make_router_inputs(case.index)
    t16 = lambda bits: torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)
    x, g, w, b = (t16(inp[k]) for k in ("hidden_states", "gamma", "router_weights", "router_bias"))
    T, H, E, K = case.n_tokens, case.hidden, case.n_experts, case.top_k
    norm = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((T, K), dtype=torch.int32, device=dev)
    aff = torch.empty((T, E), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(api.mla_router_workspace_bytes(T, H, E, K), dtype=torch.uint8, device=dev)
    call = lambda: api.mla_rmsnorm_router_topk(x, g, w, b, inp["eps"], K, case.act, norm, idx, aff, ws)
    call()
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.graph(graph, stream=cap):
        call()
    torch.cuda.current_stream(dev).wait_stream(cap)
    for _ in range(args.warmup):
        graph.replay()
    ms, _ = timed_steps(args.steps, lambda ev: graph.replay(), False)
    return ms, case


def time_tp_o_proj(dev, stream, timed_steps, args):
    """The head split's fused o-projection + reduction (mla_tp_o_proj_allreduce) on the
    block's o-projection shape (T=128, 128 heads x v_head_dim 128 = 16384 -> hidden
    7168): one rank (world 1), and a world of 8 with every rank on this GPU (n_local =
    8: the same weight bytes, eight copies of every output store). Stream launches
    (the finish kernel is a cooperative launch), L2 flushed before each; per-call ms
    lists by world."""
    import torch
    from sparse_mla_decode_front_b200 import api, tp
    from sparse_mla_decode_front_b200.device import _to_torch
    T, K, H = 128, 16384, 7168
    x = synth.make_o_proj_inputs(T, K, H, seed=7200)
    o, w = _to_torch(x["o"], True).to(dev), _to_torch(x["o_proj_w"], True).to(dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    out = {}
    for world in (1, 8):
        pb = tp.PeerBuffers.local(world, T, H, device=dev)
        epoch = [0]

        def call(ev):
            epoch[0] += 1
            api.mla_tp_o_proj_allreduce(o, w, pb.table(0, epoch[0]), world, ws, stream)
        for _ in range(args.warmup):
            call(None)
        out[world], _ = timed_steps(args.steps, call, False)
        torch.cuda.synchronize(dev)
        status = int(ws[:4].view(torch.int32).item())
        if status:
            raise RuntimeError(f"fused o-projection reduction: device status {status:#x}")
    return out


def tp_summary(ms1, ms8, plain_oproj_ms, peaks) -> dict:
    wbytes = 2 * 16384 * 7168
    return {"shape": "T=128, o [128, 16384] @ o_proj_w [16384, 7168] (128 heads x v_head_dim 128)",
            "world1_us": 1e3 * ms1, "world8_all_ranks_on_one_gpu_us": 1e3 * ms8,
            "plain_o_proj_stage_us": 1e3 * plain_oproj_ms,
            "world1_achieved_gbs": wbytes / (ms1 / 1e3) / 1e9,
            "world1_roofline_frac": wbytes / (ms1 / 1e3) / 1e9 / peaks["hbm_gbs"],
            "mode": "stream launches (projection with reduction into the owners' accumulators + cooperative "
                    "finish), L2 flushed before each",
            "note": "world 8 computes every rank's share on this one GPU in one launch of each kernel; on 8 GPUs "
                    "each rank streams 1/8 of o_proj_w and its tiles cross NVLink to their owners",
            "gpu_launches_per_call": 2}


def stage_roofline(nbytes: float, flops: float, t_s: float, peaks: dict) -> dict:
    """Roofline object of a stage timed inside the step (seconds of back-to-back kernels):
    its binding bound is the larger of bytes / copy rate and flops / sustained bf16 rate;
    achieved = those bytes or flops / t_s; the other bound's fraction beside it."""
    bw_time = nbytes / (peaks["hbm_gbs"] * 1e9)
    tc_time = flops / (peaks["bf16_tflops_sustained"] * 1e12)
    if bw_time >= tc_time:
        roof = {"bound": "hbm", "achieved": nbytes / t_s / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_kind": "copy"}
    else:
        roof = {"bound": "tensor", "achieved": flops / t_s / 1e12, "peak": peaks["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "peak_kind": "sustained bf16"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["other_bound_frac"] = min(bw_time, tc_time) / t_s
    return roof


def router_summary(case, ms_call, peaks) -> dict:
    """JSON object of the router measurement: time, algorithmic bytes, roofline."""
    from sparse_mla_decode_front_b200 import api
    T, H, E, K = case.n_tokens, case.hidden, case.n_experts, case.top_k
    # hidden in, gamma, router weights, bias; norm out, indices, affinities
    nbytes = 2 * T * H + 2 * H + 2 * H * E + 2 * E + 2 * T * H + 4 * T * K + 2 * T * E
    gbs = nbytes / (ms_call / 1e3) / 1e9
    return {"case": case.note, "us_per_call": 1e3 * ms_call, "tokens_per_s": T / (ms_call / 1e3),
            "mode": "CUDA graph of one call, replayed; L2 flushed between replays",
            "algorithmic_bytes": nbytes, "achieved_gbs": gbs, "roofline_frac": gbs / peaks["hbm_gbs"],
            "bound": "hbm", "gpu_launches_per_call": api.mla_router_launches(T, H, E, K)}


def time_workload(wl_other, dev, stream, flush, n_steps, n_warm, peaks) -> dict:
    """One other workload of the block: its step captured as a CUDA graph and replayed (L2
    flushed before each replay, CUDA events on the launching stream), and its stages from
    stream-launched steps with events inside the C call; algorithmic bytes and roofline."""
    import torch
    from sparse_mla_decode_front_b200 import _lib
    from sparse_mla_decode_front_b200.device import DecodeStep
    inp = synth.make_inputs(wl_other.index)
    d = inp["dims"]
    alg = algorithmic(inp)
    step = DecodeStep(inp, device=dev)
    for _ in range(n_warm):
        step.run(stream)
    nst = _lib.MLA_N_STAGES
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(n_steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize(dev)
    for i in range(n_steps):
        flush.zero_()
        step.run(stream, ev[i])
    torch.cuda.synchronize(dev)
    stage = [statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(n_steps)) for j in range(nst)]
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.graph(graph, stream=cap):
        step.run()
    stream.wait_stream(cap)
    for _ in range(n_warm):
        graph.replay()
    ms = []
    for _ in range(n_steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        graph.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ms.append(a.elapsed_time(b))
    status = step.device_status(stream)
    if status != 0:
        raise SystemExit(f"{wl_other.name}: device status {status:#x}")
    us = 1e3 * statistics.median(ms)
    roof_us = 1e6 * max(alg["total"]["bytes"] / (peaks["hbm_gbs"] * 1e9),
                        alg["total"]["flops"] / (peaks["bf16_tflops"] * 1e12))
    core = alg["stages"]["core"]
    core_us = 1e3 * stage[_lib.STAGE_NAMES.index("core")]
    core_roof_us = 1e6 * max(core["bytes"] / (peaks["hbm_gbs"] * 1e9),
                             core["flops"] / (peaks["bf16_tflops_sustained"] * 1e12))
    out = {"us_per_step": us, "tokens_per_s": d.n_tokens / (us / 1e6), "n_tokens": d.n_tokens,
           "n_prior": d.n_prior, "valid_keys": alg["n_valid"], "algorithmic_bytes": alg["total"]["bytes"],
           "algorithmic_flops": alg["total"]["flops"], "step_roofline_us": roof_us,
           "step_roofline_frac": roof_us / us, "achieved_hbm_gbs": alg["total"]["bytes"] / (us / 1e6) / 1e9,
           "stage_us": {n: 1e3 * v for n, v in zip(_lib.STAGE_NAMES, stage)},
           "core": {"us": core_us, "algorithmic_bytes": core["bytes"], "roofline_us": core_roof_us,
                    "roofline_frac": core_roof_us / core_us},
           "mode": f"CUDA graph of one step, replayed {n_steps} times (median), L2 flushed before each; "
                   "stages from stream-launched steps with events"}
    del step, graph
    torch.cuda.empty_cache()
    return out


def run_ours(args, wl):
    import torch
    import torch.distributed as dist

    from sparse_mla_decode_front_b200 import _lib
    from sparse_mla_decode_front_b200.device import DecodeStep

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    # Each rank decodes its own batch of sequences (its own replica of the workload).
    inp = synth.make_inputs(wl.index, seed=replica_seed(wl.index, rank))
    d = inp["dims"]
    alg = algorithmic(inp)
    step = DecodeStep(inp, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    nst = _lib.MLA_N_STAGES

    def timed_steps(n, fn, with_stages):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(n)] \
            if with_stages else None
        if ev:
            for row in ev:          # create the events before their handles are used
                for e in row:
                    e.record(stream)
        outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        torch.cuda.synchronize(dev)
        for i in range(n):
            flush.zero_()
            outer[i][0].record(stream)
            fn(ev[i] if ev else None)
            outer[i][1].record(stream)
        torch.cuda.synchronize(dev)
        ms = [a.elapsed_time(b) for a, b in outer]
        stage_ms = None
        if ev:
            stage_ms = [[row[j].elapsed_time(row[j + 1]) for row in ev] for j in range(nst)]
        return ms, stage_ms

    # nvidia-smi samples every 200 ms, so the sampling window spans warm-up (kept
    # busy for >= 0.6 s), the timed steps and the end-to-end steps.
    sampler = ClockSampler(gpu_uuid(dev))
    with sampler:
        t_end = time.perf_counter() + 0.6
        n_warm = 0
        while n_warm < args.warmup or time.perf_counter() < t_end:
            step.run(stream)
            n_warm += 1
            if n_warm >= args.warmup:
                torch.cuda.synchronize(dev)
        torch.cuda.synchronize(dev)
        if step.device_status(stream) != 0:
            raise SystemExit(f"device status {step.device_status(stream):#x} after warm-up")

        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        ms, stage_ms = timed_steps(args.steps, lambda ev: step.run(stream, ev), True)
        torch.cuda.synchronize(dev)
        n_launch = step.n_launches

        # The same step captured once as a CUDA graph and replayed: what a serving loop runs.
        graph = torch.cuda.CUDAGraph()
        capture_stream = torch.cuda.Stream(dev)   # capture needs a non-default stream
        capture_stream.wait_stream(stream)
        with torch.cuda.graph(graph, stream=capture_stream):
            step.run()
        stream.wait_stream(capture_stream)
        torch.cuda.synchronize(dev)
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        graph_ms, _ = timed_steps(args.steps, lambda ev: graph.replay(), False)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        if step.device_status(stream) != 0:
            raise SystemExit(f"device status {step.device_status(stream):#x} after graph replays")

        # The fused step stream-launched without stage events (like-for-like with the
        # separate path's stream launches).
        plain_ms, _ = timed_steps(args.steps, lambda ev: step.run(stream), False)
        # The separate-kernel path (query tiles through HBM), for the fused-vs-separate comparison:
        # stream-launched, and captured as a CUDA graph like the fused headline.
        for _ in range(args.warmup):
            step.run_separate(stream)
        sep_ms, _ = timed_steps(args.steps, lambda ev: step.run_separate(stream), False)
        sep_graph = torch.cuda.CUDAGraph()
        capture_stream.wait_stream(stream)
        with torch.cuda.graph(sep_graph, stream=capture_stream):
            step.run_separate()
        stream.wait_stream(capture_stream)
        for _ in range(args.warmup):
            sep_graph.replay()
        sep_graph_ms, _ = timed_steps(args.steps, lambda ev: sep_graph.replay(), False)
        torch.cuda.synchronize(dev)
        if step.device_status(stream) != 0:
            raise SystemExit(f"device status {step.device_status(stream):#x} after the separate path")

        # end to end through the public API: per-step inputs from pinned host memory, output
        # read back. Serial: one step at a time, L2 flushed before each. Pipelined (the e2e
        # value): back-to-back steps as a serving loop runs them, every step's copies
        # overlapped with the neighbouring steps' compute.
        step.host_buffers()
        e2e_ms, _ = timed_steps(max(3, args.steps // 2), lambda ev: step.run_from_host(stream), False)
        step.pipeline_from_host(max(3, args.warmup), stream)
        n_pipe = max(10, args.steps)
        pipe_step = step.pipeline_from_host(n_pipe, stream) / n_pipe

        # The MoE router step that follows the block in a decoder layer (fused RMSNorm +
        # router top-K), timed the same way: graph replays, L2 flushed before each.
        router_ms, router_case = time_router(dev, flush, timed_steps, args)
        # Tensor parallelism over heads: the fused o-projection + reduction on its own.
        tp_ms = time_tp_o_proj(dev, stream, timed_steps, args)
    stream_step = sum(ms) / len(ms)
    graph_step = sum(graph_ms) / len(graph_ms)
    sep_step = sum(sep_ms) / len(sep_ms)
    plain_step = sum(plain_ms) / len(plain_ms)
    sep_graph_step = sum(sep_graph_ms) / len(sep_graph_ms)
    stage_avg = [sum(s) / len(s) for s in stage_ms]
    e2e_step = sum(e2e_ms) / len(e2e_ms)
    q = lambda v, f: float(np.percentile(v, f))
    pct = [q(graph_ms, 10), q(graph_ms, 50), q(graph_ms, 90)]

    router_step = sum(router_ms) / len(router_ms)
    tp1, tp8 = (sum(tp_ms[k]) / len(tp_ms[k]) for k in (1, 8))
    ms_step, stream_step, sep_step, e2e_step, pipe_step, router_step, tp1, tp8, plain_step, sep_graph_step, *pct = \
        max_over_ranks([graph_step, stream_step, sep_step, e2e_step, pipe_step, router_step, tp1, tp8, plain_step,
                        sep_graph_step] + pct, device=dev)

    peaks = load_peaks()
    result = None
    if rank == 0:
        names = _lib.STAGE_NAMES
        top = int(np.argmax(stage_avg))
        stg = alg["stages"][names[top]]
        t_s = stage_avg[top] / 1e3
        roof = stage_roofline(stg["bytes"], stg["flops"], t_s, peaks)
        roof["traffic"] = profiled_traffic(names[top], wl.name)
        roof["kernel"] = names[top]
        roof["peak_source"] = peaks["source"]
        step_bytes = alg["total"]["bytes"]
        step_roof_us = 1e6 * max(step_bytes / (peaks["hbm_gbs"] * 1e9),
                                 alg["total"]["flops"] / (peaks["bf16_tflops"] * 1e12))
        tokens = world * d.n_tokens
        result = {
            "metric": METRIC, "value": tokens / (ms_step / 1e3), "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "us_per_step": 1e3 * ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "n_tokens": d.n_tokens, "n_heads": d.n_heads,
                       "n_prior": d.n_prior, "hidden": d.hidden, "kv_cache_rows": d.n_blocks * d.block_size,
                       "valid_keys": alg["n_valid"], "parallelism": f"dp{world}",
                       "l2": "flushed (256 MB write) before every timed step"},
            "achieved_hbm_gbs": step_bytes / (ms_step / 1e3) / 1e9,
            "step_roofline_us": step_roof_us, "step_roofline_frac": step_roof_us / (1e3 * ms_step),
            "timing": {"mode": "CUDA graph of one step, replayed; L2 flushed between replays",
                       "p10_us": 1e3 * pct[0], "p50_us": 1e3 * pct[1], "p90_us": 1e3 * pct[2],
                       "stream_launch_us_per_step": 1e3 * plain_step,
                       "stream_launch_with_stage_events_us_per_step": 1e3 * stream_step},
            "separate_path": {"graph_us_per_step": 1e3 * sep_graph_step,
                              "graph_over_fused": sep_graph_step / ms_step,
                              "stream_launch_us_per_step": 1e3 * sep_step,
                              "stream_over_fused": sep_step / plain_step,
                              "note": "mla_decode_qkv + mla_decode_attention (query tiles through HBM), timed "
                                      "both ways the fused step is: captured as a CUDA graph and replayed, and "
                                      "stream-launched without events; L2 flushed before each step"},
            "stage_us": {n: 1e3 * v for n, v in zip(names, stage_avg)},
            "roofline": roof,
            "gpu_launches": n_launch * args.steps,
            "e2e": {"value": tokens / (pipe_step / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": step.h2d_bytes(), "d2h_bytes_per_step": step.d2h_bytes(),
                    "us_per_step": 1e3 * pipe_step,
                    "mode": f"{n_pipe} back-to-back steps through the public API (the block call of each of two "
                            "buffer sets captured once as a CUDA graph and replayed): each step's "
                            "inputs copied from pinned host memory and its output read back, the copies on two "
                            "copy streams overlapped with the neighbouring steps' compute (two device buffer "
                            "sets); timed from the first upload to the last read-back",
                    "l2": ("not flushed between the back-to-back steps: each step reads "
                           f"{step_bytes / 1e6:.0f} MB (algorithmic), "
                           + ("more than the 126 MB L2" if step_bytes > 126e6 else "less than the 126 MB L2")),
                    "serial_us_per_step": 1e3 * e2e_step,
                    "serial_mode": "one step at a time (copy in, block call, copy out on one stream), "
                                   "L2 flushed before each"},
            "router_topk": router_summary(router_case, router_step, peaks),
            "tp_o_proj": tp_summary(tp1, tp8, stage_avg[-1], peaks),
            "clocks": dict(sampler.summary(), window="warm-up + timed + e2e steps"),
        }
    if rank == 0 and world == 1 and not args.no_workloads:
        # The other workloads of the block (the headline workload's own figures are above).
        del step
        torch.cuda.empty_cache()
        others = {}
        for w in synth.WORKLOADS:
            if w.name in ("tiny", wl.name):
                continue
            others[w.name] = time_workload(w, dev, stream, flush, max(5, args.steps // 2), args.warmup, peaks)
        result["workloads"] = others
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(inp, args.cpu_tokens)
    elif rank == 0:
        result["cpu_baseline"] = None
    if rank == 0:
        print(json.dumps(result), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="gather128", choices=[w.name for w in synth.WORKLOADS])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-tokens", type=int, default=32, help="tokens of the single-thread oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-workloads", action="store_true", help="skip the other workloads' figures")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    wl = synth.WORKLOAD_BY_NAME[args.workload]
    if args.impl == "reference":
        return run_reference(args, wl)
    return run_ours(args, wl)


if __name__ == "__main__":
    sys.exit(main())
