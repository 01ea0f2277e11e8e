"""ctypes binding of the C ABI (include/sparse_mla_decode.h): loading and
argument marshalling only. Every step of the block runs in the library's
CUDA kernels; there is no Python or CPU implementation behind these calls.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsparse_mla_decode.so")

MLA_OK = 0
MLA_ERR_NULL_POINTER = -1
MLA_ERR_BAD_DIMS = -2
MLA_ERR_UNSUPPORTED_DIMS = -3
MLA_ERR_MISALIGNED = -4
MLA_ERR_WORKSPACE_TOO_SMALL = -5
MLA_ERR_CUDA = -6
MLA_ERR_BAD_ARGUMENT = -7

MLA_DEV_BAD_BLOCK_ID = 0x1
MLA_DEV_BAD_LOGICAL_BLOCK = 0x2
MLA_DEV_BAD_SLOT = 0x4
MLA_DEV_WAIT_TIMEOUT = 0x8

DIM_FIELDS = ("n_tokens", "hidden", "q_lora_rank", "kv_lora_rank", "qk_nope_head_dim",
              "qk_rope_head_dim", "v_head_dim", "n_heads", "block_size", "n_blocks",
              "max_blocks_per_seq", "n_prior")


class MlaDims(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in DIM_FIELDS]


MLA_TP_MAX_WORLD = 8


class MlaTpPeers(ctypes.Structure):
    """mla_tp_peers (include/mla_tp.h): every rank's accumulator, output and counters."""
    _fields_ = [("world", ctypes.c_int32), ("rank", ctypes.c_int32), ("epoch", ctypes.c_uint32),
                ("reserved", ctypes.c_int32), ("acc", ctypes.c_void_p * MLA_TP_MAX_WORLD),
                ("out", ctypes.c_void_p * MLA_TP_MAX_WORLD), ("flags", ctypes.c_void_p * MLA_TP_MAX_WORLD)]


class MlaIpcHandle(ctypes.Structure):
    _fields_ = [("bytes", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64)]


class MlaLaunchOpts(ctypes.Structure):
    _fields_ = [("stage_events", ctypes.c_void_p), ("n_launches", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("out_f32", ctypes.c_void_p),
                ("tp", ctypes.POINTER(MlaTpPeers))]


MLA_N_STAGES = 5
MLA_NOALLOC_SCRATCH_BYTES = 8 << 20
STAGE_NAMES = ("index_resolve", "front_fold", "core", "out_absorb", "o_proj")


class MlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {status_string(code)} (code {code})"
        if code == MLA_ERR_CUDA:
            msg += f" [{lib().mla_last_cuda_error_string().decode()}]"
        super().__init__(msg)


_lib = None

# Exported entry points and their C signatures.
_VP, _FP, _IP = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
SIGNATURES = {
    "mla_abi_version": (ctypes.c_int32, []),
    "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "mla_last_cuda_error_string": (ctypes.c_char_p, []),
    "mla_block_check_dims": (ctypes.c_int, [ctypes.POINTER(MlaDims)]),
    "mla_block_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(MlaDims)]),
    "mla_get_device_status": (ctypes.c_int, [_VP, _VP, ctypes.POINTER(ctypes.c_int32)]),
    "mla_block_gather_decode": (ctypes.c_int, [_VP] * 18 + [ctypes.POINTER(MlaDims), ctypes.c_float,
                                                            ctypes.c_float, _VP, ctypes.c_size_t, _VP]),
    "mla_block_gather_decode_noalloc": (ctypes.c_int, [_VP] * 18 + [ctypes.POINTER(MlaDims), ctypes.c_float,
                                                                    ctypes.c_float, _VP]),
    "mla_block_gather_decode_noalloc_status": (ctypes.c_int, [_VP, ctypes.POINTER(ctypes.c_int32)]),
    "mla_block_gather_decode_ex": (ctypes.c_int, [_VP] * 18 + [ctypes.POINTER(MlaDims), ctypes.c_float,
                                                               ctypes.c_float, _VP, ctypes.c_size_t, _VP,
                                                               ctypes.POINTER(MlaLaunchOpts)]),
    "mla_decode_qkv": (ctypes.c_int, [_VP] * 13 + [ctypes.POINTER(MlaDims), ctypes.c_float, _VP, ctypes.c_size_t,
                                                   _VP]),
    "mla_decode_attention": (ctypes.c_int, [_VP] * 8 + [ctypes.POINTER(MlaDims), ctypes.c_float, _VP,
                                                         ctypes.c_size_t, _VP]),
    "mla_router_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 4),
    "mla_router_launches": (ctypes.c_int, [ctypes.c_int] * 4),
    "mla_rmsnorm_router_topk": (ctypes.c_int, [_VP] * 4 + [ctypes.c_int] * 4 + [ctypes.c_float, ctypes.c_int]
                                + [_VP] * 4 + [ctypes.c_size_t, _VP]),
    "mla_tp_o_proj_allreduce": (ctypes.c_int, [_VP, _VP] + [ctypes.c_int] * 3
                                + [ctypes.POINTER(MlaTpPeers), ctypes.c_int, _VP, _VP]),
    "mla_ipc_export": (ctypes.c_int, [_VP, ctypes.POINTER(MlaIpcHandle)]),
    "mla_ipc_open": (ctypes.c_int, [ctypes.POINTER(MlaIpcHandle), ctypes.POINTER(ctypes.c_void_p)]),
    "mla_ipc_close": (ctypes.c_int, [_VP]),
}
MLA_ROUTER_SIGMOID = 0
MLA_ROUTER_SOFTMAX = 1


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m sparse_mla_decode_front_b200.build`")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(l, name)
            fn.restype = res
            fn.argtypes = args
        _lib = l
    return _lib


def status_string(code: int) -> str:
    return lib().mla_status_string(int(code)).decode()


def make_dims(**kw) -> MlaDims:
    return MlaDims(*[int(kw[f]) for f in DIM_FIELDS])
