"""Independent GPU cross-check of the three GEMMs against a library kernel.

cuBLASLt's MXFP8 GEMM (torch's scaled_mm: E4M3 operands, one UE8M0 scale per
1x32 block, FP32 accumulation, BF16 out) is fed this library's own quantized
operands.  Each 1x128 (or 128x128) scale byte is repeated over the four
32-element sub-blocks it covers, which gives exactly the same real-valued
operands, so both kernels compute the same exact sum of exactly representable
products and differ only in FP32 summation order and the final BF16 rounding
(block-scaled FP8 linear layer spec: FP32 accumulation, BF16 output; the MX
sub-block replication is the reading of the pages' "MXFP8 path" remark).

Each result must lie within 4e-3 * rms + 1 BF16 ulp of the exact product, so
the two may differ element-wise by up to twice that, and their relative
Frobenius difference must stay below 1e-3.  The test also pins the blocked
scale layout of include/puro_fp8.h to the MX scale-factor layout the library
kernel reads (a layout error would scramble the scales and fail by far).
"""
import numpy as np
import pytest
import torch

from helpers import bf16_ulp, unblock

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_block_scaled_13_b200 as m
    from fp8_block_scaled_13_b200 import build
    build.build()
    return m


def _scaled_mm():
    import torch.nn.functional as F
    if not hasattr(F, "scaled_mm") or not hasattr(torch, "float8_e8m0fnu"):
        pytest.skip("torch has no MXFP8 scaled_mm")
    return F


def _mx_scales(s_rg: np.ndarray) -> torch.Tensor:
    """[R, G] UE8M0 bytes of 128-wide groups -> the MX (1x32) scale array in
    the 128x4 swizzled layout, each byte repeated for its four sub-blocks."""
    R, G = s_rg.shape
    Rp = (R + 127) // 128 * 128
    s = np.full((Rp, G), 127, dtype=np.uint8)
    s[:R] = s_rg
    r = np.arange(Rp)[:, None, None]
    g32 = 4 * np.arange(G)[None, :, None] + np.arange(4)[None, None, :]
    g4 = G  # ceil(4G / 4) chunks of 4 sub-blocks per 128-row block
    idx = ((r // 128) * g4 + g32 // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + g32 % 4
    mx = np.empty(Rp * G * 4, dtype=np.uint8)
    mx[idx.reshape(-1)] = np.broadcast_to(s[:, :, None], (Rp, G, 4)).reshape(-1)
    return torch.from_numpy(mx).cuda().view(torch.float8_e8m0fnu)


def _library(F, qa, sa_rg, qb, sb_rg):
    """C[m, n] = sum_k A[m, k] B[n, k] from E4M3 codes and per-128 scale bytes."""
    a = qa.contiguous().view(torch.float8_e4m3fn)
    b = qb.contiguous().view(torch.float8_e4m3fn)
    return F.scaled_mm(a, b.t(), _mx_scales(sa_rg), F.ScalingType.BlockWise1x32,
                       _mx_scales(sb_rg), F.ScalingType.BlockWise1x32,
                       swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                       swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                       output_dtype=torch.bfloat16)


def _assert_agree(ours: torch.Tensor, lib: torch.Tensor, what: str):
    a = ours.float().cpu().numpy().astype(np.float64)
    b = lib.float().cpu().numpy().astype(np.float64)
    den = np.linalg.norm(b)
    rel = np.linalg.norm(a - b) / den
    assert rel <= 1e-3, "%s: relative Frobenius difference %.3g" % (what, rel)
    rms = np.sqrt(np.mean(b ** 2))
    excess = np.abs(a - b) - 2.0 * (4e-3 * rms + bf16_ulp(np.maximum(np.abs(a), np.abs(b))))
    assert excess.max() <= 0.0, "%s: an element differs by %.3g beyond the bound" % (what, excess.max())
    return rel


@pytest.mark.parametrize("m,n,k", [(256, 384, 512), (1024, 640, 1024)])
def test_gemms_agree_with_library_mxfp8(fp8, m, n, k):
    F = _scaled_mm()
    g = torch.Generator().manual_seed(11)
    x = torch.randn(m, k, generator=g)
    x[torch.rand(m, k, generator=g) < 1e-3] *= 100.0  # outliers: varied scales across groups
    x = x.to(torch.bfloat16).cuda()
    w = (torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16).cuda()
    dy = (torch.randn(m, n, generator=g) * 1e-3).to(torch.bfloat16).cuda()
    xq = fp8.quant_act(x, "both")
    dyq = fp8.quant_act(dy, "both")
    wq = fp8.quant_weight(w)
    y = fp8.gemm_fprop(xq, wq)
    dx = fp8.gemm_dgrad(dyq, wq)
    dw = fp8.gemm_wgrad(dyq, xq)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0

    kb, nb, mb = k // 128, n // 128, m // 128
    lib_y = _library(F, xq.q, unblock(xq.s, m, kb), wq.q, unblock(wq.s_fwd, n, kb))
    lib_dx = _library(F, dyq.q, unblock(dyq.s, m, nb), wq.qt, unblock(wq.s_bwd, k, nb))
    lib_dw = _library(F, dyq.qt[:, :m], unblock(dyq.st, n, mb), xq.qt[:, :m], unblock(xq.st, k, mb))
    torch.cuda.synchronize()
    _assert_agree(y, lib_y, "fprop")
    _assert_agree(dx, lib_dx, "dgrad")
    _assert_agree(dw, lib_dw, "wgrad")
