"""bench.py's accounting, checked on the CPU: the algorithmic work it divides
by measured time (FLOPs per GEMM launch, bytes per quantizer launch) and the
mixed-precision MFU bookkeeping.  The expected values are written out from the
definitions (2*M*N*K per GEMM; BF16 in, E4M3 codes and UE8M0 scale bytes out),
not taken from the code under test."""
import math

import torch

import bench
from fp8_block_scaled_13_b200.inputs import Linear, Workload


def _attn_proj_shapes():
    """The bench workload's shapes on the meta device (no data)."""
    meta = dict(dtype=torch.bfloat16, device="meta")
    m = 8192
    layers = []
    for name, n, k in (("qkv", 3072, 2048), ("o_proj", 2048, 2048)):
        layers.append(Linear(name, torch.empty(m, k, **meta), torch.empty(n, k, **meta),
                             torch.empty(m, n, **meta)))
    return Workload("attn_proj", 1, layers)


def test_gemm_flops_per_launch():
    costs = bench._unit_costs(_attn_proj_shapes())
    # the per-layer GFLOP figures of the attention-projection config: QKV 103.1, O 68.7
    assert costs["qkv.fprop"] == ("flops", 2 * 8192 * 3072 * 2048)
    assert abs(costs["qkv.fprop"][1] / 1e9 - 103.08) < 0.01
    assert abs(costs["o_proj.fprop"][1] / 1e9 - 68.72) < 0.01
    # one launch computes dgrad and wgrad: twice the fprop work
    assert costs["qkv.dgrad_wgrad"] == ("flops", 2 * costs["qkv.fprop"][1])
    assert costs["o_proj.dgrad_wgrad"] == ("flops", 2 * costs["o_proj.fprop"][1])
    # the step's FLOPs (the numerator of `value`) are the sum over its GEMM launches
    wl = _attn_proj_shapes()
    assert sum(v for kind, v in costs.values() if kind == "flops") == wl.gemm_flops()


def test_quantizer_bytes_per_launch():
    costs = bench._unit_costs(_attn_proj_shapes())
    # BOTH layouts: 2 B read, two 1-B codes and two scale bytes per 128 values
    assert costs["qkv.quant_x"] == ("bytes", 8192 * 2048 * 2 + 2 * 8192 * 2048 + 2 * 8192 * 2048 // 128)
    assert math.isclose(costs["qkv.quant_x"][1] / (8192 * 2048), 4.015625)
    assert costs["qkv.quant_dy"][1] == 8192 * 3072 * 4 + 2 * 8192 * 3072 // 128
    # weight: 2 B read, codes and transposed codes, one compact scale per 128x128 block
    assert costs["qkv.quant_weight"] == ("bytes", 3072 * 2048 * 4 + 24 * 16)


def _full_block_shapes(m):
    meta = dict(dtype=torch.bfloat16, device="meta")
    layers = []
    for name, n, k in (("qkv", 3072, 2048), ("o_proj", 2048, 2048), ("gate_up", 12288, 2048),
                       ("down", 2048, 6144)):
        layers.append(Linear(name, torch.empty(m, k, **meta), torch.empty(n, k, **meta),
                             torch.empty(m, n, **meta)))
    return Workload("full_block", 4, layers)


def test_full_block_flops_per_step():
    # fwd + bwd of the block: 3 GEMMs x 2*M*N*K per layer; at M = 32768,
    # 6 * 32768 * (3072*2048 + 2048*2048 + 12288*2048 + 2048*6144) = 9.483 TFLOP
    wl = _full_block_shapes(32768)
    assert wl.gemm_flops() == 6 * 32768 * (3072 * 2048 + 2048 * 2048 + 12288 * 2048 + 2048 * 6144)
    assert abs(wl.gemm_flops() / 1e12 - 9.4833) < 1e-3
    # the per-M figures of the sweep: 1.185 / 2.315 / 4.742 TFLOP at M = 4096 / 8000 / 16384
    for m, tf in ((4096, 1.1854), (8000, 2.3153), (16384, 4.7416)):
        assert abs(_full_block_shapes(m).gemm_flops() / 1e12 - tf) < 1e-3
    costs = bench._unit_costs(wl)
    assert costs["gate_up.dgrad_wgrad"] == ("flops", 4 * 32768 * 12288 * 2048)
    assert costs["down.quant_x"] == ("bytes", 32768 * 6144 * 4 + 2 * 32768 * 6144 // 128)


def test_input_sets_cover_three_l2_capacities():
    # 132 MB per attention-projection set: three sets; the 2.2 GB block: one
    assert bench.n_input_sets(_attn_proj_shapes()) == 3
    assert bench.n_input_sets(_full_block_shapes(32768)) == 1
    assert bench.input_set_bytes(_full_block_shapes(32768)) == 2 * (
        32768 * (2048 * 3 + 6144) + 32768 * (3072 + 2048 + 12288 + 2048)
        + (3072 * 2048 + 2048 * 2048 + 12288 * 2048 + 2048 * 6144))


def test_clock_summary_uses_loaded_samples():
    idle = ["0", "1965", "1965", "120", "0", "Not Active", "Not Active", "Not Active", "Not Active"]
    busy = ["0", "1800", "1965", "990", "100", "Not Active", "Not Active", "Not Active", "Active"]
    busy2 = ["0", "1700", "1965", "1000", "98", "Not Active", "Not Active", "Not Active", "Active"]
    out = bench.summarize_clocks([idle, busy, busy2, idle])
    assert out["sm_mhz"] == 1750.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples_under_load"] == 2
    # no loaded sample: fall back to all samples
    out = bench.summarize_clocks([idle])
    assert out["sm_mhz"] == 1965.0 and out["reasons"] == []


def test_mfu_accounting_closed_forms():
    peaks = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6516.0}
    # at the measured peaks themselves the MFU against them is exactly 1
    out = bench.mfu_accounting(2800.0, 1400.0, peaks)
    assert math.isclose(out["mfu_vs_measured"], 1.0, abs_tol=1e-4)
    # P_eff is the time-weighted mean: 1 / (0.72 / 2800 + 0.28 / 1400) = 2187.5
    assert math.isclose(out["p_eff_measured"], 2187.5, abs_tol=0.05)
    # nominal dense peaks 4500 (FP8) and 2250 (BF16): 1 / (0.72/4500 + 0.28/2250) = 3515.6
    assert math.isclose(out["p_eff_nominal"], 3515.6, abs_tol=0.05)
    # a worked case: 1800 TF/s FP8 and 1270 TF/s BF16 project to 1611.7 TF/s, 0.7368 of P_eff
    out = bench.mfu_accounting(1800.0, 1270.0, peaks)
    assert math.isclose(out["projected_tflops"], 1611.7, abs_tol=0.05)
    assert math.isclose(out["mfu_vs_measured"], 0.7368, abs_tol=1e-4)


def test_gemm_peak_regime():
    # a short run at full clock: the burst peak
    assert bench.gemm_peak({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}, 3180.0, 2800.0) == (
        3180.0, "burst")
    # power cap active but the clock held up: still burst
    assert bench.gemm_peak({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]},
                           3180.0, 2800.0)[1] == "burst"
    # a long power-capped run at 1.1 GHz: the sustained peak
    assert bench.gemm_peak({"sm_mhz": 1100.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]},
                           3180.0, 2800.0) == (2800.0, "sustained")
    # no clock record: burst
    assert bench.gemm_peak({"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]},
                           3180.0, 2800.0)[1] == "burst"
