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
