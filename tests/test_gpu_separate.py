"""The separate-kernel path (mla_decode_qkv, then mla_decode_attention, query
tiles through HBM) against the fp64 oracle and against the fused block.

Page "MLA Attention Block Gather Decode Kernel API Reference" (introduction and
"Notes") contrasts the fused block with separate QKV and attention kernels; the
two paths compute the same step, so the bars are the fused path's: cache rows
within 1 bf16 ulp of the oracle's, output max|err| / max|oracle| <= 1e-2.
"""
import numpy as np
import pytest
import torch

from sparse_mla_decode_front_b200 import api, synth
from sparse_mla_decode_front_b200.device import DecodeStep
from test_gpu_parity import OUT_TOL, ROW_ULPS, oracle_run, ulp_distance

pytestmark = pytest.mark.gpu


def separate_run(inp):
    step = DecodeStep(inp)
    out = step.run_separate()
    torch.cuda.synchronize()
    d = inp["dims"]
    cache = step.t["kv_cache"].view(-1, d.kv_row_dim)
    slots = torch.from_numpy(inp["slot_mapping"].astype(np.int64)).cuda()
    rows = cache[slots].view(torch.int16).cpu().numpy().view(np.uint16)
    return out.float().cpu().numpy().astype(np.float64), rows, step


@pytest.mark.parametrize("wl,tokens", [(0, None), (1, None), (3, [0, 37, 64, 127])])
def test_separate_path_matches_oracle(wl, tokens):
    inp = synth.make_inputs(wl)
    y, rows, step = separate_run(inp)
    assert step.device_status() == 0
    y_ref, rows_ref = oracle_run(inp, tokens)
    assert ulp_distance(rows, rows_ref).max() <= ROW_ULPS
    sel = slice(None) if tokens is None else list(tokens)
    err = np.abs(y[sel] - y_ref).max() / np.abs(y_ref).max()
    assert err <= OUT_TOL, f"output rel err {err:.3e}"


def test_separate_path_matches_fused():
    # Same kernels on both paths; they differ only in where the query tiles live.
    # The split-K reductions add partial sums in run-dependent order, so the fp32
    # outputs agree to rounding, not bit for bit, and their bf16 roundings can land
    # one ulp apart: up to 2^-8 of the largest magnitude, under the 2^-7 bar.
    inp = synth.make_inputs(1)
    step = DecodeStep(inp)
    y_sep = step.run_separate().float().clone()
    q_sep = step.q_tiles.clone()
    y_fused = step.run().float()
    torch.cuda.synchronize()
    assert (y_sep - y_fused).abs().max().item() <= 2.0 ** -7 * y_fused.abs().max().item()
    d = inp["dims"]
    assert q_sep.shape == (d.n_tokens, d.n_heads, d.kv_lora_rank + d.qk_rope_head_dim)
    assert torch.isfinite(q_sep.float()).all()
    assert step.device_status() == 0


def test_separate_path_rejects_wrong_q_tiles_shape():
    inp = synth.make_inputs(0)
    step = DecodeStep(inp)
    t = step.t
    bad = torch.empty(3, 3, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError, match="q_tiles"):
        api.mla_decode_attention(bad, t["kv_cache"], t["block_table"], t["positions"], t["gather_indices"],
                                 t["out_absorb_w"], t["o_proj_w"], step.out, step.dims, step.scale,
                                 step.workspace)
