"""Host-side helpers of bench.py: the roofline object of the dominant stage, the
algorithmic bytes and flops it is computed from, and the profiled-traffic lookup."""
import math

import bench
from sparse_mla_decode_front_b200 import synth

PEAKS = {"hbm_gbs": 6531.9, "bf16_tflops": 1618.5, "bf16_tflops_sustained": 1371.3, "source": "measured"}


def test_core_of_gather128_is_tensor_bound_at_the_sustained_rate():
    # The core of gather128: 262144 kept rows x 1152 B plus the 18.9 MB query tiles, and
    # 2 h (R + L) flops per kept key with h = 128, R = 576, L = 512.
    rows = 128 * 2048
    nbytes = rows * 1152 + 128 * 128 * 576 * 2
    flops = rows * 2 * 128 * (576 + 512)
    roof = bench.stage_roofline(nbytes, flops, 150e-6, PEAKS)
    assert roof["bound"] == "tensor" and roof["peak"] == PEAKS["bf16_tflops_sustained"]
    assert math.isclose(roof["achieved"], flops / 150e-6 / 1e12)
    assert math.isclose(roof["frac"], flops / (PEAKS["bf16_tflops_sustained"] * 1e12) / 150e-6)
    assert math.isclose(roof["other_bound_frac"], nbytes / (PEAKS["hbm_gbs"] * 1e9) / 150e-6)
    assert roof["other_bound_frac"] < roof["frac"]
    # at the burst rate the same stage would have read as HBM-bound: the sustained rate decides
    assert nbytes / (PEAKS["hbm_gbs"] * 1e9) > flops / (PEAKS["bf16_tflops"] * 1e12)


def test_weight_stream_is_hbm_bound():
    # o_proj of gather128: 234.9 MB of weights, 2 x 128 x 16384 x 7168 flops
    nbytes, flops = 16384 * 7168 * 2, 2 * 128 * 16384 * 7168
    roof = bench.stage_roofline(nbytes, flops, 45e-6, PEAKS)
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert math.isclose(roof["achieved"], nbytes / 45e-6 / 1e9)
    assert roof["frac"] == roof["achieved"] / PEAKS["hbm_gbs"]


def test_algorithmic_totals_of_gather128():
    # every weight once + every kept row + cache-row writes + hidden in/out + index tensors
    inp = synth.make_inputs(synth.WORKLOAD_BY_NAME["gather128"].index)
    alg = bench.algorithmic(inp)
    d = inp["dims"]
    weights = 2 * (d.hidden * d.q_lora_rank + d.hidden * d.kv_row_dim + d.q_lora_rank * d.n_heads * d.qk_head_dim
                   + d.n_heads * d.qk_nope_head_dim * d.kv_lora_rank + d.n_heads * d.v_head_dim * d.kv_lora_rank
                   + d.n_heads * d.v_head_dim * d.hidden)
    assert alg["stages"]["core"]["bytes"] >= 128 * 2048 * 1152
    assert alg["total"]["bytes"] > weights + 128 * 2048 * 1152
    assert 6.7e8 < alg["total"]["bytes"] < 6.9e8          # the 681 MB of the step roofline
    assert 1.19e11 < alg["total"]["flops"] < 1.23e11      # ~121 GFLOP


def test_profiled_traffic_follows_the_source_hash():
    # a stage without a recorded summary has no traffic; the core's is read while its
    # source still has the recorded hash
    assert bench.profiled_traffic("o_proj", "gather128") is None
    t = bench.profiled_traffic("core", "gather128")
    assert t is None or t > 300e6
