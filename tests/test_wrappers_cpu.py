"""Host-side argument handling of the torch-facing wrappers, with no GPU.

Every check runs before the first call into the library, so these tests
neither need a device nor load libpuro_fp8.so.
"""
import pytest
import torch

import fp8_block_scaled_13_b200 as fp8


def _act(dev, rows=128, cols=128):
    return fp8.QuantAct(rows, cols,
                        q=torch.zeros(rows, cols, dtype=torch.uint8, device=dev),
                        s=torch.zeros(512, dtype=torch.uint8, device=dev))


def _weight(dev, n=128, k=128):
    return fp8.QuantWeight(n, k,
                           torch.zeros(n, k, dtype=torch.uint8, device=dev),
                           torch.zeros(n // 128, k // 128, dtype=torch.uint8, device=dev),
                           s_fwd=torch.zeros(512, dtype=torch.uint8, device=dev))


def test_operands_on_different_devices_are_refused():
    with pytest.raises(ValueError, match="different devices"):
        fp8.gemm_fprop(_act("cpu"), _weight("meta"))
    with pytest.raises(ValueError, match="different devices"):
        fp8.quant_act(torch.zeros(128, 128, dtype=torch.bfloat16), out=_act("meta"))


def test_host_tensors_are_refused_before_any_launch():
    with pytest.raises(ValueError, match="CUDA"):
        fp8.quant_act(torch.zeros(128, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        fp8.quant_weight(torch.zeros(128, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        fp8.gemm_fprop(_act("cpu"), _weight("cpu"))


def test_shape_and_layout_errors():
    with pytest.raises(ValueError, match="inner dimensions"):
        fp8.gemm_fprop(_act("cpu", cols=256), _weight("cpu", k=128))
    with pytest.raises(ValueError, match="row-wise"):
        fp8.gemm_fprop(fp8.QuantAct(128, 128), _weight("cpu"))
    with pytest.raises(ValueError, match="transposed"):
        fp8.gemm_dgrad(_act("cpu"), _weight("cpu"))
    with pytest.raises(ValueError, match="accumulate"):
        fp8.gemm_wgrad(fp8.QuantAct(128, 128, qt=torch.zeros(128, 128, dtype=torch.uint8)),
                       fp8.QuantAct(128, 128, qt=torch.zeros(128, 128, dtype=torch.uint8)),
                       accumulate=True)

