"""The C-ABI library: it loads, exports every declared entry point, and its
host-side validation rejects bad calls before touching a GPU."""
import ctypes
import glob
import os
import re

import pytest

from sparse_mla_decode_front_b200 import _lib, api, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(mla_\w+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    l = _lib.lib()
    names = declared_functions()
    assert "mla_block_gather_decode" in names
    for n in names:
        assert hasattr(l, n), n
    assert set(names) <= set(_lib.SIGNATURES), "binding lacks a signature"


def test_status_strings_and_version():
    assert api.mla_abi_version() >> 16 == 1
    for c in range(-7, 1):
        assert api.mla_status_string(c) and "unknown" not in api.mla_status_string(c)
    assert "unknown" in api.mla_status_string(-99)
    # no CUDA call has failed on this host thread
    assert _lib.lib().mla_last_cuda_error_string().decode() == "no error"


def test_dims_validation():
    d = synth.workload_dims(3)
    assert api.mla_block_check_dims(d) == 0
    assert api.mla_block_workspace_bytes(d) > 0
    for field, v, code in [("hidden", 0, _lib.MLA_ERR_BAD_DIMS), ("qk_rope_head_dim", 63, _lib.MLA_ERR_BAD_DIMS),
                           ("n_heads", -1, _lib.MLA_ERR_BAD_DIMS), ("n_tokens", -1, _lib.MLA_ERR_BAD_DIMS),
                           ("kv_lora_rank", 500, _lib.MLA_ERR_UNSUPPORTED_DIMS)]:
        bad = dict(d.__dict__, **{field: v})
        assert api.mla_block_check_dims(bad) == code, field
        assert api.mla_block_workspace_bytes(bad) == 0


def _call(dims, ptrs=None, ws_bytes=1 << 30, scale=0.1, eps=1e-6, gather=0x1000):
    l = _lib.lib()
    p = [ctypes.c_void_p(0x1000 + 256 * i) for i in range(18)] if ptrs is None else ptrs
    p[16] = ctypes.c_void_p(gather)
    d = _lib.make_dims(**dims)
    return l.mla_block_gather_decode(*p, ctypes.byref(d), ctypes.c_float(scale), ctypes.c_float(eps),
                                     ctypes.c_void_p(0x100000), ctypes.c_size_t(ws_bytes), None)


def test_host_side_rejections():
    # None of these reach the GPU: validation returns first.
    d = dict(synth.workload_dims(0).__dict__)
    p = [ctypes.c_void_p(0x1000 + 256 * i) for i in range(18)]
    p[3] = ctypes.c_void_p(0)
    assert _call(d, p) == _lib.MLA_ERR_NULL_POINTER
    p = [ctypes.c_void_p(0x1000 + 256 * i) for i in range(18)]
    p[5] = ctypes.c_void_p(0x1008)
    assert _call(d, p) == _lib.MLA_ERR_MISALIGNED
    assert _call(d, ws_bytes=16) == _lib.MLA_ERR_WORKSPACE_TOO_SMALL
    assert _call(d, scale=float("nan")) == _lib.MLA_ERR_BAD_ARGUMENT
    assert _call(d, eps=-1.0) == _lib.MLA_ERR_BAD_ARGUMENT
    assert _call(d, gather=0) == _lib.MLA_ERR_NULL_POINTER
    assert _call(dict(d, hidden=0)) == _lib.MLA_ERR_BAD_DIMS
    # an empty batch is a no-op, even with no buffers at all
    nulls = [ctypes.c_void_p(0)] * 18
    assert _call(dict(d, n_tokens=0), nulls, ws_bytes=0, gather=0) == _lib.MLA_OK
    l = _lib.lib()
    assert l.mla_get_device_status(None, None, None) == _lib.MLA_ERR_NULL_POINTER


def test_python_binding_rejects_host_tensors():
    import torch
    with pytest.raises(ValueError, match="CUDA"):
        api._check("hidden_states", torch.zeros(2, 4, dtype=torch.bfloat16), torch.bfloat16)


def test_separate_entry_points_host_side_rejections():
    # mla_decode_qkv / mla_decode_attention validate before any CUDA call.
    l = _lib.lib()
    d = _lib.make_dims(**synth.workload_dims(0).__dict__)
    ws = ctypes.c_void_p(0x100000)

    def qkv(p, ws_bytes=1 << 30, eps=1e-6):
        return l.mla_decode_qkv(*p, ctypes.byref(d), ctypes.c_float(eps), ws, ctypes.c_size_t(ws_bytes), None)

    def att(p, ws_bytes=1 << 30, scale=0.1):
        return l.mla_decode_attention(*p, ctypes.byref(d), ctypes.c_float(scale), ws, ctypes.c_size_t(ws_bytes),
                                      None)

    good13 = lambda: [ctypes.c_void_p(0x1000 + 256 * i) for i in range(13)]
    good8 = lambda: [ctypes.c_void_p(0x1000 + 256 * i) for i in range(8)]
    p = good13()
    p[12] = ctypes.c_void_p(0)                       # q_tiles
    assert qkv(p) == _lib.MLA_ERR_NULL_POINTER
    p = good13()
    p[12] = ctypes.c_void_p(0x1004)
    assert qkv(p) == _lib.MLA_ERR_MISALIGNED
    assert qkv(good13(), ws_bytes=16) == _lib.MLA_ERR_WORKSPACE_TOO_SMALL
    assert qkv(good13(), eps=float("inf")) == _lib.MLA_ERR_BAD_ARGUMENT
    p = good8()
    p[4] = ctypes.c_void_p(0)                        # gather_indices with n_prior > 0
    assert att(p) == _lib.MLA_ERR_NULL_POINTER
    p = good8()
    p[0] = ctypes.c_void_p(0x1002)                   # q_tiles
    assert att(p) == _lib.MLA_ERR_MISALIGNED
    assert att(good8(), scale=float("nan")) == _lib.MLA_ERR_BAD_ARGUMENT
    assert att(good8(), ws_bytes=0) == _lib.MLA_ERR_WORKSPACE_TOO_SMALL
    bad = _lib.make_dims(**dict(synth.workload_dims(0).__dict__, hidden=0))
    assert l.mla_decode_qkv(*good13(), ctypes.byref(bad), ctypes.c_float(1e-6), ws, ctypes.c_size_t(1 << 30),
                            None) == _lib.MLA_ERR_BAD_DIMS


def test_router_workspace_and_host_side_rejections():
    l = _lib.lib()
    assert l.mla_router_workspace_bytes(128, 7168, 256, 8) > 0
    for dims in [(128, 7168, 32, 8), (128, 7168, 2048, 8), (128, 7160, 256, 8), (128, 7168, 256, 0),
                 (128, 7168, 256, 33), (-1, 7168, 256, 8), (128, 7168, 250, 8)]:
        assert l.mla_router_workspace_bytes(*dims) == 0, dims
        assert l.mla_router_launches(*dims) == 0, dims
    # one cooperative launch where the device allows it, else prep, projection and finish
    assert l.mla_router_launches(128, 7168, 256, 8) in (1, 3)
    assert l.mla_router_launches(16, 1024, 512, 8) == 3
    p = [ctypes.c_void_p(0x1000 + 256 * i) for i in range(8)]

    def call(T=4, H=256, E=64, K=4, eps=1e-6, act=0, ptrs=p, bias=None, ws=1 << 20):
        return l.mla_rmsnorm_router_topk(ptrs[0], ptrs[1], ptrs[2], bias, T, H, E, K, ctypes.c_float(eps), act,
                                         ptrs[3], ptrs[4], ptrs[5], ptrs[6], ctypes.c_size_t(ws), None)
    assert call(T=0) == _lib.MLA_OK   # nothing to do
    assert call(H=0) == _lib.MLA_ERR_BAD_DIMS
    assert call(E=48) == _lib.MLA_ERR_UNSUPPORTED_DIMS
    assert call(K=65) == _lib.MLA_ERR_UNSUPPORTED_DIMS
    assert call(act=2) == _lib.MLA_ERR_BAD_ARGUMENT
    assert call(eps=float("nan")) == _lib.MLA_ERR_BAD_ARGUMENT
    q = list(p)
    q[0] = ctypes.c_void_p(0)
    assert call(ptrs=q) == _lib.MLA_ERR_NULL_POINTER
    q = list(p)
    q[3] = ctypes.c_void_p(0x1008)
    assert call(ptrs=q) == _lib.MLA_ERR_MISALIGNED
    assert call(bias=ctypes.c_void_p(0x1004)) == _lib.MLA_ERR_MISALIGNED
    assert call(ws=16) == _lib.MLA_ERR_WORKSPACE_TOO_SMALL


def _peers(world=2, rank=0, epoch=1, base=0x200000):
    t = _lib.MlaTpPeers()
    t.world, t.rank, t.epoch = world, rank, epoch
    for r in range(min(max(world, 0), _lib.MLA_TP_MAX_WORLD)):
        t.acc[r], t.out[r], t.flags[r] = base + 0x1000 * r, base + 0x100000 + 0x1000 * r, base + 0x200000 + 64 * r
    return t


def test_tp_host_side_rejections():
    l = _lib.lib()
    o, w, ws = ctypes.c_void_p(0x1000), ctypes.c_void_p(0x2000), ctypes.c_void_p(0x100000)

    def call(tp, T=4, k=256, H=512, n_local=1, o=o, w=w, ws=ws):
        return l.mla_tp_o_proj_allreduce(o, w, T, k, H, None if tp is None else ctypes.byref(tp), n_local, ws,
                                         None)
    assert call(None) == _lib.MLA_ERR_NULL_POINTER
    assert call(_peers(), T=0) == _lib.MLA_ERR_BAD_DIMS
    assert call(_peers(), k=24) == _lib.MLA_ERR_UNSUPPORTED_DIMS
    assert call(_peers(), H=512 + 32) == _lib.MLA_ERR_UNSUPPORTED_DIMS   # 544 is not a multiple of 64
    for bad in [_peers(world=0), _peers(world=9), _peers(rank=2), _peers(rank=-1), _peers(epoch=0)]:
        assert call(bad) == _lib.MLA_ERR_BAD_ARGUMENT
    assert call(_peers(world=4, rank=1), n_local=2) == _lib.MLA_ERR_BAD_ARGUMENT    # rank not a multiple
    assert call(_peers(world=4, rank=0), n_local=3) == _lib.MLA_ERR_BAD_ARGUMENT    # world not a multiple
    t = _peers()
    t.flags[1] = None
    assert call(t) == _lib.MLA_ERR_NULL_POINTER
    t = _peers()
    t.acc[1] = 0x200008
    assert call(t) == _lib.MLA_ERR_MISALIGNED
    assert call(_peers(), o=ctypes.c_void_p(0)) == _lib.MLA_ERR_NULL_POINTER
    assert call(_peers(), ws=ctypes.c_void_p(0x100010)) == _lib.MLA_ERR_MISALIGNED
    # the block call: a peer table excludes out_f32, and is validated like the above
    opts = _lib.MlaLaunchOpts()
    opts.tp = ctypes.pointer(_peers(epoch=0))
    p = [ctypes.c_void_p(0x1000 + 256 * i) for i in range(18)]
    d = _lib.make_dims(**synth.workload_dims(0).__dict__)
    blk = lambda: l.mla_block_gather_decode_ex(*p, ctypes.byref(d), ctypes.c_float(0.1), ctypes.c_float(1e-6),
                                               ctypes.c_void_p(0x100000), ctypes.c_size_t(1 << 30), None,
                                               ctypes.byref(opts))
    assert blk() == _lib.MLA_ERR_BAD_ARGUMENT
    opts.tp = ctypes.pointer(_peers())
    opts.out_f32 = ctypes.c_void_p(0x3000)
    assert blk() == _lib.MLA_ERR_BAD_ARGUMENT


def test_ipc_host_side_rejections():
    l = _lib.lib()
    h = _lib.MlaIpcHandle()
    assert l.mla_ipc_export(None, ctypes.byref(h)) == _lib.MLA_ERR_NULL_POINTER
    assert l.mla_ipc_export(ctypes.c_void_p(0x1000), None) == _lib.MLA_ERR_NULL_POINTER
    p = ctypes.c_void_p()
    assert l.mla_ipc_open(None, ctypes.byref(p)) == _lib.MLA_ERR_NULL_POINTER
    assert l.mla_ipc_open(ctypes.byref(h), None) == _lib.MLA_ERR_NULL_POINTER
    assert l.mla_ipc_close(None) == _lib.MLA_ERR_NULL_POINTER


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library every entry point raises; nothing falls back to a
    Python or CPU implementation."""
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libsparse_mla_decode.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    with pytest.raises(ImportError):
        _lib.lib()
    with pytest.raises(ImportError):
        api.mla_abi_version()
    with pytest.raises(ImportError):
        api.mla_block_workspace_bytes(synth.make_inputs(0)["dims"])
