"""The allocation-free entry point, mla_block_gather_decode_noalloc.

It serves callers that cannot allocate device memory (a plugin inside an
engine that owns all device memory through its own pool, or code that must
not call the allocator while it builds a stream): the step's scratch is a
fixed array inside the library instead of a caller workspace. These tests call
it through the C ABI and compare it with mla_block_gather_decode (which takes
a workspace) on the same inputs, over two calls in a row, with the parity
tolerance of the other GPU tests. This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_mla_decode_front_b200 import _lib, api, synth
from sparse_mla_decode_front_b200.device import DecodeStep, upload

pytestmark = pytest.mark.gpu

OUT_TOL = 1e-2


def _noalloc(t, out, inp, stream):
    d = _lib.make_dims(**{f: getattr(inp["dims"], f) for f in _lib.DIM_FIELDS})
    ptrs = [ctypes.c_void_p(t[k].data_ptr()) for k in api.ARG_ORDER[:-1]] + [ctypes.c_void_p(out.data_ptr())]
    return _lib.lib().mla_block_gather_decode_noalloc(
        *ptrs, ctypes.byref(d), ctypes.c_float(inp["softmax_scale"]), ctypes.c_float(inp["norm_eps"]),
        ctypes.c_void_p(stream.cuda_stream))


@pytest.mark.parametrize("workload", [0, 1])
def test_noalloc_matches_workspace_entry_point(workload):
    inp = synth.make_inputs(workload)
    d = inp["dims"]
    assert api.mla_block_workspace_bytes(d) <= _lib.MLA_NOALLOC_SCRATCH_BYTES
    ref_step = DecodeStep(inp)
    ref = ref_step.run().float().clone()
    torch.cuda.synchronize()
    assert ref_step.device_status() == 0
    ref_rows = ref_step.t["kv_cache"].view(-1, d.kv_row_dim)[torch.from_numpy(inp["slot_mapping"].astype(np.int64)).cuda()]

    t = upload(inp)                                  # fresh tensors, fresh cache
    out = torch.empty(d.n_tokens, d.hidden, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    scale = ref.abs().max().item()
    for call in range(2):
        out.fill_(float("nan"))
        assert _noalloc(t, out, inp, stream) == _lib.MLA_OK, call
        torch.cuda.synchronize()
        err = (out.float() - ref).abs().max().item() / scale
        assert err <= OUT_TOL, f"call {call}: rel err {err:.3e}"
        rows = t["kv_cache"].view(-1, d.kv_row_dim)[torch.from_numpy(inp["slot_mapping"].astype(np.int64)).cuda()]
        assert torch.equal(rows.view(torch.int16), ref_rows.view(torch.int16)), call


def test_noalloc_rejects_sizes_beyond_its_scratch():
    inp = synth.make_inputs(0)
    big = synth.workload_dims(3)
    assert api.mla_block_workspace_bytes(big) > _lib.MLA_NOALLOC_SCRATCH_BYTES
    t = upload(inp)
    out = torch.empty(2, 256, dtype=torch.bfloat16, device="cuda")
    d = _lib.make_dims(**{f: getattr(big, f) for f in _lib.DIM_FIELDS})
    ptrs = [ctypes.c_void_p(t[k].data_ptr()) for k in api.ARG_ORDER[:-1]] + [ctypes.c_void_p(out.data_ptr())]
    rc = _lib.lib().mla_block_gather_decode_noalloc(*ptrs, ctypes.byref(d), ctypes.c_float(0.1),
                                                    ctypes.c_float(1e-6), None)
    assert rc == _lib.MLA_ERR_WORKSPACE_TOO_SMALL


def _noalloc_status(stream):
    st = ctypes.c_int32(-1)
    assert _lib.lib().mla_block_gather_decode_noalloc_status(ctypes.c_void_p(stream.cuda_stream),
                                                             ctypes.byref(st)) == _lib.MLA_OK
    return st.value


def test_noalloc_status_word_reports_device_errors():
    # The step's device status bits live in the built-in array; the getter reads them
    # back: a bad slot is flagged (and its row not written), and the next clean call
    # clears the word again.
    inp = synth.make_inputs(0)
    d = inp["dims"]
    t = upload(inp)
    out = torch.empty(d.n_tokens, d.hidden, dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    bad = dict(inp)
    bad["slot_mapping"] = inp["slot_mapping"].copy()
    bad["slot_mapping"][1] = -4
    tb = upload(bad)
    assert _noalloc(tb, out, bad, stream) == _lib.MLA_OK
    assert _noalloc_status(stream) & _lib.MLA_DEV_BAD_SLOT
    assert _noalloc(t, out, inp, stream) == _lib.MLA_OK
    assert _noalloc_status(stream) == 0