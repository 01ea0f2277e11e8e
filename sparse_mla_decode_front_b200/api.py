"""Python binding of the C ABI, with the same entry-point names.

Argument marshalling only: torch tensors are checked (device, dtype,
contiguity, shape) and their device pointers handed to the library; torch
provides device memory and streams and nothing else. Every step of the block
runs in the library's CUDA kernels.

The page-style call ``mla_attention_block_gather_decode`` (page "MLA
Attention Block Gather Decode Kernel API Reference", section "API Reference")
infers the dimensions from tensor shapes as the page does and allocates the
output and the scratch workspace with torch.
"""
from __future__ import annotations

import ctypes
from typing import Dict, Optional

import torch

from . import _lib
from ._lib import MlaDims, MlaError, make_dims

BF16_ARGS = ("hidden_states", "wq_a", "wq_b", "wkv_a", "q_absorb_w", "out_absorb_w", "o_proj_w",
             "kv_cache")
F32_ARGS = ("input_norm_w", "q_norm_w", "kv_norm_w", "cos", "sin")
I32_ARGS = ("slot_mapping", "block_table", "positions", "gather_indices")
ARG_ORDER = ("hidden_states", "input_norm_w", "wq_a", "q_norm_w", "wq_b", "wkv_a", "kv_norm_w",
             "q_absorb_w", "out_absorb_w", "o_proj_w", "cos", "sin", "kv_cache", "slot_mapping",
             "block_table", "positions", "gather_indices", "out")


def _dims_struct(dims) -> MlaDims:
    if isinstance(dims, MlaDims):
        return dims
    if isinstance(dims, dict):
        return make_dims(**dims)
    return make_dims(**{f: getattr(dims, f) for f in _lib.DIM_FIELDS})


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def mla_status_string(code: int) -> str:
    return _lib.status_string(code)


def mla_abi_version() -> int:
    return int(_lib.lib().mla_abi_version())


def mla_block_check_dims(dims) -> int:
    d = _dims_struct(dims)
    return int(_lib.lib().mla_block_check_dims(ctypes.byref(d)))


def mla_block_workspace_bytes(dims) -> int:
    d = _dims_struct(dims)
    return int(_lib.lib().mla_block_workspace_bytes(ctypes.byref(d)))


def mla_get_device_status(workspace: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int32(0)
    rc = _lib.lib().mla_get_device_status(ctypes.c_void_p(workspace.data_ptr()),
                                          ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(v))
    if rc != 0:
        raise MlaError(rc, "mla_get_device_status")
    return int(v.value)


def _check(name: str, t: Optional[torch.Tensor], dtype, shape=None, allow_none=False):
    if t is None:
        if allow_none:
            return
        raise ValueError(f"{name} is None")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def expected_shapes(d) -> Dict[str, tuple]:
    g = lambda f: getattr(d, f) if not isinstance(d, dict) else d[f]
    T, H, Lq, L = g("n_tokens"), g("hidden"), g("q_lora_rank"), g("kv_lora_rank")
    dn, dr, dv, h = g("qk_nope_head_dim"), g("qk_rope_head_dim"), g("v_head_dim"), g("n_heads")
    bs, nb, mb, P = g("block_size"), g("n_blocks"), g("max_blocks_per_seq"), g("n_prior")
    return dict(hidden_states=(T, H), input_norm_w=(1, H), wq_a=(H, Lq), q_norm_w=(1, Lq),
                wq_b=(Lq, h * (dn + dr)), wkv_a=(H, L + dr), kv_norm_w=(1, L),
                q_absorb_w=(h, dn, L), out_absorb_w=(h, dv, L), o_proj_w=(h * dv, H),
                cos=(T, dr // 2), sin=(T, dr // 2), kv_cache=(nb, 1, bs, L + dr),
                slot_mapping=(T,), block_table=(T, mb), positions=(T,), gather_indices=(T, P),
                out=(T, H))


def mla_block_gather_decode(hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w,
                            q_absorb_w, out_absorb_w, o_proj_w, cos, sin, kv_cache, slot_mapping,
                            block_table, positions, gather_indices, out, dims, softmax_scale: float,
                            norm_eps: float, workspace: torch.Tensor, stream=None,
                            stage_events=None, out_f32: Optional[torch.Tensor] = None,
                            tp: Optional[_lib.MlaTpPeers] = None) -> int:
    """Enqueue one block step on ``stream`` (default: torch's current stream).

    Tensors as in the C header; gammas may be [1, n] or [n]. ``stage_events``
    (optional) is a list of MLA_N_STAGES + 1 torch.cuda.Event recorded at the
    stage boundaries. ``out_f32`` (optional, [T, hidden] fp32): the o-projection's
    fp32 sums are written there instead of ``out`` (which may then be None).
    ``tp`` (optional, an MlaTpPeers table): the weights are rank ``tp.rank``'s head
    shard and the call leaves the all-ranks bf16 output in ``tp.out[tp.rank]``
    (``out`` is not used). Returns the number of kernels enqueued. Raises MlaError with the library's
    code on failure.
    """
    args = dict(hidden_states=hidden_states, input_norm_w=input_norm_w, wq_a=wq_a, q_norm_w=q_norm_w,
                wq_b=wq_b, wkv_a=wkv_a, kv_norm_w=kv_norm_w, q_absorb_w=q_absorb_w,
                out_absorb_w=out_absorb_w, o_proj_w=o_proj_w, cos=cos, sin=sin, kv_cache=kv_cache,
                slot_mapping=slot_mapping, block_table=block_table, positions=positions,
                gather_indices=gather_indices, out=out)
    d = _dims_struct(dims)
    shapes = expected_shapes(d)
    for k, v in args.items():
        dt = torch.bfloat16 if (k in BF16_ARGS or k == "out") else \
            torch.float32 if k in F32_ARGS else torch.int32
        shp = shapes[k]
        if k in ("input_norm_w", "q_norm_w", "kv_norm_w") and v is not None and v.dim() == 1:
            shp = shp[1:]
        _check(k, v, dt, shp, allow_none=(k == "gather_indices" and d.n_prior == 0) or
               (k == "out" and (out_f32 is not None or tp is not None)))
    _check("workspace", workspace, torch.uint8)
    _check("out_f32", out_f32, torch.float32, shapes["out"], allow_none=True)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else 0)
    opts = _lib.MlaLaunchOpts()
    if out_f32 is not None:
        opts.out_f32 = ptr(out_f32)
    if tp is not None:
        opts.tp = ctypes.pointer(tp)
    ev_arr = None
    if stage_events is not None:
        if len(stage_events) != _lib.MLA_N_STAGES + 1:
            raise ValueError(f"stage_events needs {_lib.MLA_N_STAGES + 1} events")
        ev_arr = (ctypes.c_void_p * len(stage_events))(*[e.cuda_event for e in stage_events])
        opts.stage_events = ctypes.cast(ev_arr, ctypes.c_void_p)
    rc = _lib.lib().mla_block_gather_decode_ex(
        *[ptr(args[k]) for k in ARG_ORDER], ctypes.byref(d), ctypes.c_float(softmax_scale),
        ctypes.c_float(norm_eps), ptr(workspace), ctypes.c_size_t(workspace.numel()),
        ctypes.c_void_p(_stream_handle(stream)), ctypes.byref(opts))
    if rc != 0:
        raise MlaError(rc, "mla_block_gather_decode")
    return int(opts.n_launches)


def _check_args(args: dict, d: MlaDims, extra_shapes: Dict[str, tuple] = None):
    shapes = dict(expected_shapes(d), **(extra_shapes or {}))
    for k, v in args.items():
        dt = torch.bfloat16 if (k in BF16_ARGS or k in ("out", "q_tiles")) else \
            torch.float32 if k in F32_ARGS else torch.int32
        shp = shapes[k]
        if k in ("input_norm_w", "q_norm_w", "kv_norm_w") and v is not None and v.dim() == 1:
            shp = shp[1:]
        _check(k, v, dt, shp, allow_none=(k == "gather_indices" and d.n_prior == 0))


def q_tiles_shape(d) -> tuple:
    """Shape of the query tiles handed from mla_decode_qkv to mla_decode_attention."""
    d = _dims_struct(d)
    return (d.n_tokens, d.n_heads, d.kv_lora_rank + d.qk_rope_head_dim)


def mla_decode_qkv(hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w, q_absorb_w,
                   cos, sin, kv_cache, slot_mapping, q_tiles, dims, norm_eps: float,
                   workspace: torch.Tensor, stream=None) -> None:
    """Separate path, first half: front-fold into ``q_tiles`` [T, h, L + dr] (bf16) and this
    step's cache rows. Enqueued on ``stream``; raises MlaError on failure."""
    args = dict(hidden_states=hidden_states, input_norm_w=input_norm_w, wq_a=wq_a, q_norm_w=q_norm_w,
                wq_b=wq_b, wkv_a=wkv_a, kv_norm_w=kv_norm_w, q_absorb_w=q_absorb_w, cos=cos, sin=sin,
                kv_cache=kv_cache, slot_mapping=slot_mapping, q_tiles=q_tiles)
    d = _dims_struct(dims)
    _check_args(args, d, {"q_tiles": q_tiles_shape(d)})
    _check("workspace", workspace, torch.uint8)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = _lib.lib().mla_decode_qkv(*[ptr(v) for v in args.values()], ctypes.byref(d), ctypes.c_float(norm_eps),
                                   ptr(workspace), ctypes.c_size_t(workspace.numel()),
                                   ctypes.c_void_p(_stream_handle(stream)))
    if rc != 0:
        raise MlaError(rc, "mla_decode_qkv")


def mla_decode_attention(q_tiles, kv_cache, block_table, positions, gather_indices, out_absorb_w, o_proj_w,
                         out, dims, softmax_scale: float, workspace: torch.Tensor, stream=None) -> None:
    """Separate path, second half: index resolve, sparse latent attention of ``q_tiles``
    over the kept cache rows, out absorption and o-projection into ``out`` [T, hidden]."""
    args = dict(q_tiles=q_tiles, kv_cache=kv_cache, block_table=block_table, positions=positions,
                gather_indices=gather_indices, out_absorb_w=out_absorb_w, o_proj_w=o_proj_w, out=out)
    d = _dims_struct(dims)
    _check_args(args, d, {"q_tiles": q_tiles_shape(d)})
    _check("workspace", workspace, torch.uint8)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else 0)
    rc = _lib.lib().mla_decode_attention(*[ptr(v) for v in args.values()], ctypes.byref(d),
                                         ctypes.c_float(softmax_scale), ptr(workspace),
                                         ctypes.c_size_t(workspace.numel()),
                                         ctypes.c_void_p(_stream_handle(stream)))
    if rc != 0:
        raise MlaError(rc, "mla_decode_attention")


def dims_from_tensors(hidden_states, wq_a, wq_b, out_absorb_w, kv_cache, block_table,
                      gather_indices, n_heads, qk_nope_head_dim, qk_rope_head_dim,
                      kv_lora_rank) -> Dict[str, int]:
    """The page's dimension inference: everything not passed as an int comes from shapes."""
    T, H = hidden_states.shape
    return dict(n_tokens=T, hidden=H, q_lora_rank=wq_a.shape[1], kv_lora_rank=kv_lora_rank,
                qk_nope_head_dim=qk_nope_head_dim, qk_rope_head_dim=qk_rope_head_dim,
                v_head_dim=out_absorb_w.shape[1], n_heads=n_heads, block_size=kv_cache.shape[2],
                n_blocks=kv_cache.shape[0], max_blocks_per_seq=block_table.shape[1],
                n_prior=gather_indices.shape[1])


def mla_attention_block_gather_decode(hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a,
                                      kv_norm_w, q_absorb_w, out_absorb_w, o_proj_w, cos, sin,
                                      kv_cache, slot_mapping, block_table, positions,
                                      gather_indices, n_heads: int, qk_nope_head_dim: int,
                                      qk_rope_head_dim: int, kv_lora_rank: int,
                                      softmax_scale: float, norm_eps: float = 1e-6,
                                      workspace: Optional[torch.Tensor] = None, stream=None):
    """Page-signature call: returns out [n_tokens, hidden] bf16; mutates kv_cache."""
    dims = dims_from_tensors(hidden_states, wq_a, wq_b, out_absorb_w, kv_cache, block_table,
                             gather_indices, n_heads, qk_nope_head_dim, qk_rope_head_dim,
                             kv_lora_rank)
    rc = mla_block_check_dims(dims)
    if rc != 0:
        raise MlaError(rc, "mla_block_check_dims")
    need = mla_block_workspace_bytes(dims)
    if workspace is None or workspace.numel() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=hidden_states.device)
    out = torch.empty(dims["n_tokens"], dims["hidden"], dtype=torch.bfloat16, device=hidden_states.device)
    mla_block_gather_decode(hidden_states, input_norm_w, wq_a, q_norm_w, wq_b, wkv_a, kv_norm_w,
                            q_absorb_w, out_absorb_w, o_proj_w, cos, sin, kv_cache, slot_mapping,
                            block_table, positions, gather_indices, out, dims, softmax_scale,
                            norm_eps, workspace, stream)
    return out


# ---------------------------------------------------------------------------
# Fused RMSNorm + router top-K (include/moe_router.h)
# ---------------------------------------------------------------------------

ROUTER_ACTS = {"sigmoid": _lib.MLA_ROUTER_SIGMOID, "softmax": _lib.MLA_ROUTER_SOFTMAX}


def mla_router_workspace_bytes(n_tokens: int, hidden: int, n_experts: int, top_k: int) -> int:
    return int(_lib.lib().mla_router_workspace_bytes(int(n_tokens), int(hidden), int(n_experts), int(top_k)))


def mla_router_launches(n_tokens: int, hidden: int, n_experts: int, top_k: int) -> int:
    return int(_lib.lib().mla_router_launches(int(n_tokens), int(hidden), int(n_experts), int(top_k)))


def mla_rmsnorm_router_topk(hidden_states, gamma, router_weights, router_bias, eps: float, top_k: int, act: str,
                            norm_out, topk_idx, affinities, workspace, stream=None) -> None:
    """The C call on caller-allocated outputs (shapes as in include/moe_router.h);
    raises MlaError on a refused call."""
    T, H = int(hidden_states.shape[0]), int(hidden_states.shape[1])
    E = int(router_weights.shape[1])
    _check("hidden_states", hidden_states, torch.bfloat16, (T, H))
    _check("gamma", gamma, torch.bfloat16, (H,))
    _check("router_weights", router_weights, torch.bfloat16, (H, E))
    _check("router_bias", router_bias, torch.bfloat16, (E,), allow_none=True)
    _check("norm_out", norm_out, torch.bfloat16, (T, H))
    _check("topk_idx", topk_idx, torch.int32, (T, int(top_k)))
    _check("affinities", affinities, torch.bfloat16, (T, E))
    _check("workspace", workspace, torch.uint8)
    if act not in ROUTER_ACTS:
        raise ValueError(f"router activation must be one of {sorted(ROUTER_ACTS)}, got {act!r}")
    ptr = lambda t: ctypes.c_void_p(t.data_ptr() if t is not None else 0)
    rc = _lib.lib().mla_rmsnorm_router_topk(
        ptr(hidden_states), ptr(gamma), ptr(router_weights), ptr(router_bias), T, H, E, int(top_k),
        ctypes.c_float(eps), ROUTER_ACTS[act], ptr(norm_out), ptr(topk_idx), ptr(affinities), ptr(workspace),
        ctypes.c_size_t(workspace.numel()), ctypes.c_void_p(_stream_handle(stream)))
    if rc != 0:
        raise MlaError(rc, "mla_rmsnorm_router_topk")


def rmsnorm_router_topk(hidden_states, gamma, router_weights, router_bias=None, eps: float = 1e-6, top_k: int = 1,
                        router_act_fn: str = "sigmoid", stream=None):
    """Page-style call (``rmsnorm_router_topk_a2av``): hidden_states [B, S, H] or [T, H]
    bf16, gamma [1, H] or [H], router_weights [H, E], optional router_bias [1, E] or [E];
    returns (norm [T, H] bf16, top-K indices [T, K] int32, masked affinities [T, E] bf16)."""
    H = int(hidden_states.shape[-1])
    x = hidden_states.reshape(-1, H)
    T, E = int(x.shape[0]), int(router_weights.shape[1])
    dev = x.device
    norm = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((T, int(top_k)), dtype=torch.int32, device=dev)
    aff = torch.empty((T, E), dtype=torch.bfloat16, device=dev)
    nbytes = mla_router_workspace_bytes(T, H, E, top_k)
    if nbytes == 0:
        raise MlaError(_lib.MLA_ERR_UNSUPPORTED_DIMS, "mla_router_workspace_bytes")
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    mla_rmsnorm_router_topk(x.contiguous(), gamma.reshape(H), router_weights,
                            None if router_bias is None else router_bias.reshape(E), eps, top_k,
                            router_act_fn.lower(), norm, idx, aff, ws, stream)
    return norm, idx, aff


def mla_tp_o_proj_allreduce(o: torch.Tensor, o_proj_w: torch.Tensor, tp: "_lib.MlaTpPeers", n_local: int,
                            workspace: torch.Tensor, stream=None) -> None:
    """The head split's fused o-projection + reduction (include/mla_tp.h) for ranks
    [tp.rank, tp.rank + n_local): ``o`` [T, n_local * k_rank] bf16 and ``o_proj_w``
    [n_local * k_rank, hidden] bf16, the local ranks' slices side by side; every
    rank's bf16 output lands in ``tp.out[r]``."""
    if o.dim() != 2 or o_proj_w.dim() != 2 or n_local < 1 or o.shape[1] % n_local:
        raise ValueError("o must be [T, n_local * k_rank] and o_proj_w [n_local * k_rank, hidden]")
    T, k_rank, hidden = o.shape[0], o.shape[1] // n_local, o_proj_w.shape[1]
    _check("o", o, torch.bfloat16, (T, n_local * k_rank))
    _check("o_proj_w", o_proj_w, torch.bfloat16, (n_local * k_rank, hidden))
    _check("workspace", workspace, torch.uint8)
    rc = _lib.lib().mla_tp_o_proj_allreduce(
        ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(o_proj_w.data_ptr()), T, k_rank, hidden,
        ctypes.byref(tp), int(n_local), ctypes.c_void_p(workspace.data_ptr()),
        ctypes.c_void_p(_stream_handle(stream)))
    if rc != 0:
        raise MlaError(rc, "mla_tp_o_proj_allreduce")


def mla_ipc_export(t: torch.Tensor) -> bytes:
    """CUDA IPC description of the allocation holding ``t`` (handle bytes + offset),
    as bytes another process passes to mla_ipc_open."""
    h = _lib.MlaIpcHandle()
    rc = _lib.lib().mla_ipc_export(ctypes.c_void_p(t.data_ptr()), ctypes.byref(h))
    if rc != 0:
        raise MlaError(rc, "mla_ipc_export")
    return bytes(h)


def mla_ipc_open(blob: bytes) -> int:
    """Map another process's export into this one; returns the device address."""
    h = _lib.MlaIpcHandle.from_buffer_copy(blob)
    p = ctypes.c_void_p()
    rc = _lib.lib().mla_ipc_open(ctypes.byref(h), ctypes.byref(p))
    if rc != 0:
        raise MlaError(rc, "mla_ipc_open")
    return int(p.value)


def mla_ipc_close(address: int) -> None:
    rc = _lib.lib().mla_ipc_close(ctypes.c_void_p(address))
    if rc != 0:
        raise MlaError(rc, "mla_ipc_close")
