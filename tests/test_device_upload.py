"""Host-side residency helpers, exercised on the CPU device."""
import numpy as np
import torch

from sparse_mla_decode_front_b200 import api, synth
from sparse_mla_decode_front_b200.device import upload


def test_upload_bit_exact_on_cpu():
    inp = synth.make_inputs(0)
    t = upload(inp, "cpu")
    shapes = api.expected_shapes(inp["dims"])
    for k in api.BF16_ARGS:
        assert t[k].dtype == torch.bfloat16, k
        bits = t[k].view(torch.int16).numpy().view(np.uint16)
        np.testing.assert_array_equal(bits.reshape(inp[k].shape), inp[k])
    for k in api.F32_ARGS:
        assert t[k].dtype == torch.float32
    for k in api.I32_ARGS:
        assert t[k].dtype == torch.int32
    for k, shp in shapes.items():
        if k != "out":
            assert tuple(t[k].shape) == tuple(shp), k
