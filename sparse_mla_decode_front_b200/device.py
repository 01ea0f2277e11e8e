"""Device residency of a decode step's tensors (torch memory + streams only).

``upload`` places a workload's tensors in HBM: weights, gammas and index
tensors as-is, the paged cache as a zero-filled pool into which the filled
rows are scattered. ``DecodeStep`` keeps them resident with the output and
workspace buffers and runs the C-ABI call, either from device-resident inputs
or from pinned host copies of the per-step inputs (hidden states, RoPE tables
and index tensors), reading the output back to the host.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np
import torch

from . import api

PER_STEP_INPUTS = ("hidden_states", "cos", "sin", "slot_mapping", "block_table", "positions",
                   "gather_indices")


def _to_torch(a: np.ndarray, bf16: bool) -> torch.Tensor:
    """numpy -> torch; ``bf16`` arrays are uint16/int16 bit patterns viewed as bfloat16."""
    if bf16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a))


def upload(inp: Dict[str, object], device="cuda") -> Dict[str, torch.Tensor]:
    out = {}
    for k in api.BF16_ARGS:
        if k == "kv_cache":
            continue
        out[k] = _to_torch(inp[k], True).to(device)
    for k in api.F32_ARGS + api.I32_ARGS:
        out[k] = _to_torch(inp[k], False).to(device)
    d = inp["dims"]
    cache = torch.zeros(d.n_blocks, 1, d.block_size, d.kv_row_dim, dtype=torch.bfloat16, device=device)
    fill = inp["cache_fill_rows"]
    if len(fill):
        flat = inp["kv_cache"].reshape(-1, d.kv_row_dim)
        vals = _to_torch(flat[fill], True).to(device)
        cache.view(-1, d.kv_row_dim)[torch.from_numpy(fill).to(device)] = vals
    out["kv_cache"] = cache
    return out


class DecodeStep:
    """Resident tensors + workspace for repeated block steps of one workload."""

    def __init__(self, inp: Dict[str, object], device="cuda"):
        self.inp = inp
        self.dims = inp["dims"]
        self.device = torch.device(device)
        self.t = upload(inp, self.device)
        d = self.dims
        self.out = torch.empty(d.n_tokens, d.hidden, dtype=torch.bfloat16, device=self.device)
        nbytes = api.mla_block_workspace_bytes(d)
        if nbytes == 0:
            raise api.MlaError(api.mla_block_check_dims(d), "mla_block_workspace_bytes")
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self.scale = float(inp["softmax_scale"])
        self.eps = float(inp["norm_eps"])
        self._host = None

    def run(self, stream=None, stage_events=None) -> torch.Tensor:
        t = self.t
        self.n_launches = api.mla_block_gather_decode(
            t["hidden_states"], t["input_norm_w"], t["wq_a"], t["q_norm_w"], t["wq_b"], t["wkv_a"],
            t["kv_norm_w"], t["q_absorb_w"], t["out_absorb_w"], t["o_proj_w"], t["cos"], t["sin"],
            t["kv_cache"], t["slot_mapping"], t["block_table"], t["positions"], t["gather_indices"],
            self.out, self.dims, self.scale, self.eps, self.workspace, stream, stage_events)
        return self.out

    def run_separate(self, stream=None) -> torch.Tensor:
        """The same step through the separate entry points (query tiles through HBM)."""
        t = self.t
        if getattr(self, "q_tiles", None) is None:
            self.q_tiles = torch.empty(api.q_tiles_shape(self.dims), dtype=torch.bfloat16, device=self.device)
        api.mla_decode_qkv(t["hidden_states"], t["input_norm_w"], t["wq_a"], t["q_norm_w"], t["wq_b"], t["wkv_a"],
                           t["kv_norm_w"], t["q_absorb_w"], t["cos"], t["sin"], t["kv_cache"], t["slot_mapping"],
                           self.q_tiles, self.dims, self.eps, self.workspace, stream)
        api.mla_decode_attention(self.q_tiles, t["kv_cache"], t["block_table"], t["positions"],
                                 t["gather_indices"], t["out_absorb_w"], t["o_proj_w"], self.out, self.dims,
                                 self.scale, self.workspace, stream)
        return self.out

    def device_status(self, stream=None) -> int:
        return api.mla_get_device_status(self.workspace, stream)

    # --- end to end: per-step inputs from pinned host memory, output back to host
    def host_buffers(self):
        if self._host is None:
            h = {k: self.t[k].cpu().pin_memory() for k in PER_STEP_INPUTS}
            h["out"] = torch.empty(self.out.shape, dtype=self.out.dtype).pin_memory()
            self._host = h
        return self._host

    def h2d_bytes(self) -> int:
        return sum(self.t[k].numel() * self.t[k].element_size() for k in PER_STEP_INPUTS)

    def d2h_bytes(self) -> int:
        return self.out.numel() * self.out.element_size()

    def run_from_host(self, stream=None, stage_events=None) -> torch.Tensor:
        h = self.host_buffers()
        s = stream if stream is not None else torch.cuda.current_stream(self.device)
        with torch.cuda.stream(s):
            for k in PER_STEP_INPUTS:
                self.t[k].copy_(h[k], non_blocking=True)
            self.run(s, stage_events)
            h["out"].copy_(self.out, non_blocking=True)
        return h["out"]

    def _call_on(self, st, stream) -> None:
        """The block call on the per-step inputs and output of buffer set ``st``."""
        t = self.t
        api.mla_block_gather_decode(
            st["hidden_states"], t["input_norm_w"], t["wq_a"], t["q_norm_w"], t["wq_b"], t["wkv_a"],
            t["kv_norm_w"], t["q_absorb_w"], t["out_absorb_w"], t["o_proj_w"], st["cos"], st["sin"],
            t["kv_cache"], st["slot_mapping"], st["block_table"], st["positions"], st["gather_indices"],
            st["out"], self.dims, self.scale, self.eps, self.workspace, stream)

    def pipeline_from_host(self, n_steps: int, stream=None, graphs: bool = True) -> float:
        """``n_steps`` back-to-back steps end to end, as a serving loop runs them: every
        step's inputs are copied from pinned host memory and its output read back, the
        copies overlapped with the neighbouring steps' compute (step i + 1's inputs
        upload on one copy stream and step i - 1's output downloads on another while
        step i runs on ``stream``; two device buffer sets alternate). With ``graphs``
        each buffer set's block call is captured once as a CUDA graph and replayed.
        Returns the milliseconds from the first upload to the last read-back."""
        h = self.host_buffers()
        comp = stream if stream is not None else torch.cuda.current_stream(self.device)
        if getattr(self, "_pipe", None) is None:
            sets = [{k: torch.empty_like(self.t[k]) for k in PER_STEP_INPUTS} for _ in range(2)]
            for st in sets:
                st["out"] = torch.empty_like(self.out)
            self._pipe = (sets, [torch.empty_like(h["out"]).pin_memory() for _ in range(2)],
                          torch.cuda.Stream(self.device), torch.cuda.Stream(self.device))
            self._pipe_graphs = None
        sets, host_out, up, down = self._pipe
        if graphs and self._pipe_graphs is None:
            cap = torch.cuda.Stream(self.device)   # capture needs a non-default stream
            cap.wait_stream(comp)
            gs = []
            for st in sets:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap):
                    self._call_on(st, cap)
                gs.append(g)
            comp.wait_stream(cap)
            self._pipe_graphs = gs
        loaded = [torch.cuda.Event() for _ in range(2)]
        computed = [torch.cuda.Event() for _ in range(2)]
        read = [torch.cuda.Event() for _ in range(2)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        up.wait_stream(comp)
        down.wait_stream(comp)
        start.record(up)
        for i in range(n_steps):
            b = i % 2
            st = sets[b]
            if i >= 2:
                up.wait_event(computed[b])        # step i - 2 no longer reads these inputs
            with torch.cuda.stream(up):
                for k in PER_STEP_INPUTS:
                    st[k].copy_(h[k], non_blocking=True)
            loaded[b].record(up)
            comp.wait_event(loaded[b])
            if i >= 2:
                comp.wait_event(read[b])          # step i - 2's output has been read back
            if graphs:
                with torch.cuda.stream(comp):
                    self._pipe_graphs[b].replay()
            else:
                self._call_on(st, comp)
            computed[b].record(comp)
            down.wait_event(computed[b])
            with torch.cuda.stream(down):
                host_out[b].copy_(st["out"], non_blocking=True)
            read[b].record(down)
        end.record(down)
        end.synchronize()
        comp.wait_stream(up)
        comp.wait_stream(down)
        self.pipe_last_out = host_out[(n_steps - 1) % 2]   # the last step's output, on the host
        return start.elapsed_time(end)
