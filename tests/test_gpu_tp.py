"""Tensor parallelism over heads on one GPU: the ranks of a world of 2 run one
after the other on the same device (no rank waits on another), each writing its
fp32 partial (mla_launch_opts.out_f32); their sum, rounded once to bf16, meets the
block's bar against the fp64 oracle and agrees with the all-heads call."""
import numpy as np
import pytest
import torch

from sparse_mla_decode_front_b200 import synth, tp
from sparse_mla_decode_front_b200.device import DecodeStep
from test_gpu_parity import OUT_TOL, oracle_run

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("wl,tokens", [(0, None), (2, [0, 13, 31])])
def test_head_shards_on_one_gpu(wl, tokens):
    inp = synth.make_inputs(wl)
    world = 2
    ranks = [tp.TPDecodeStep(inp, r, world) for r in range(world)]
    total = sum(rk.partial().clone() for rk in ranks)
    torch.cuda.synchronize()
    assert all(rk.device_status() == 0 for rk in ranks)
    y = total.to(torch.bfloat16).float().cpu().numpy().astype(np.float64)
    y_ref, _ = oracle_run(inp, tokens)
    sel = slice(None) if tokens is None else list(tokens)
    assert np.abs(y[sel] - y_ref).max() / np.abs(y_ref).max() <= OUT_TOL
    full = DecodeStep(inp).run().float()
    torch.cuda.synchronize()
    y_full = full.cpu().numpy().astype(np.float64)
    assert np.abs(y - y_full).max() <= 2.0 ** -7 * np.abs(y_full).max()
