"""Weight gradient with an FP32 result: dW = dY^T X, and dW += dY^T X into an
FP32 gradient buffer (the pages keep gradients in FP32 while the GEMMs run in
E4M3: paperlayer.ai Appendix C, FP8 implementation pipeline).

Tolerance: the GEMM spec's -- relative Frobenius error <= 1e-3 and every
element within 4e-3 * rms(ref) of the FP64 oracle -- with one FP32 ulp of the
expected value in place of the BF16 ulp, because nothing is rounded to BF16.
"""
import numpy as np
import pytest
import torch

from helpers import assert_f32_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_block_scaled_13_b200 as m
    from fp8_block_scaled_13_b200 import build
    build.build()
    return m


def _operands(m, n, k, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(m, k, generator=g).to(torch.bfloat16)
    dy = (torch.randn(m, n, generator=g) * 1e-3).to(torch.bfloat16)
    return x, dy


def _quant(fp8, x, dy):
    return fp8.quant_act(x.cuda(), "colwise"), fp8.quant_act(dy.cuda(), "colwise")


def _check(got, ref64, init=None, what=""):
    assert_f32_close(got, ref64, init, what)


@pytest.mark.parametrize("m,n,k", [(300, 384, 512), (129, 256, 384), (1, 128, 128), (520, 640, 256)])
def test_wgrad_f32_overwrite(fp8, oracle_mod, m, n, k):
    x, dy = _operands(m, n, k, 11 + m)
    xq, dyq = _quant(fp8, x, dy)
    dw = torch.full((n, k), 5.0, dtype=torch.float32, device="cuda")
    fp8.gemm_wgrad(dyq, xq, out=dw)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    _check(dw, oracle_mod.linear_wgrad(dy, x), what="wgrad f32")


@pytest.mark.parametrize("m,n,k", [(300, 384, 512), (257, 256, 256)])
def test_wgrad_f32_accumulate(fp8, oracle_mod, m, n, k):
    x, dy = _operands(m, n, k, 23 + m)
    xq, dyq = _quant(fp8, x, dy)
    ref = oracle_mod.linear_wgrad(dy, x)
    g = torch.Generator().manual_seed(3)
    init = (torch.randn(n, k, generator=g) * float(np.sqrt(np.mean(ref ** 2)))).float()
    dw = init.cuda()
    fp8.gemm_wgrad(dyq, xq, out=dw, accumulate=True)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    _check(dw, ref, init.numpy(), "wgrad += (once)")
    # a second micro-batch with the same operands: init + 2 dY^T X
    fp8.gemm_wgrad(dyq, xq, out=dw, accumulate=True)
    torch.cuda.synchronize()
    _check(dw, 2 * ref, init.numpy(), "wgrad += (twice)")


def test_wgrad_f32_accumulate_is_deterministic(fp8):
    x, dy = _operands(520, 640, 384, 31)
    xq, dyq = _quant(fp8, x, dy)
    init = torch.randn(640, 384, generator=torch.Generator().manual_seed(4)).cuda()
    outs = []
    for _ in range(2):
        dw = init.clone()
        fp8.gemm_wgrad(dyq, xq, out=dw, accumulate=True)
        fp8.gemm_wgrad(dyq, xq, out=dw, accumulate=True)
        outs.append(dw)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1])


def test_wgrad_f32_rounds_to_the_bf16_result(fp8):
    """Same MMA stream, same accumulation order: the FP32 result rounded to
    BF16 (RNE) is bit-identical to the BF16 output."""
    x, dy = _operands(1000, 384, 640, 41)
    xq, dyq = _quant(fp8, x, dy)
    d32 = torch.empty(384, 640, dtype=torch.float32, device="cuda")
    fp8.gemm_wgrad(dyq, xq, out=d32)
    d16 = fp8.gemm_wgrad(dyq, xq)
    torch.cuda.synchronize()
    assert torch.equal(d32.to(torch.bfloat16).view(torch.int16), d16.view(torch.int16))


def test_wgrad_f32_zero_tokens(fp8):
    x = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    xq, dyq = fp8.quant_act(x, "colwise"), fp8.quant_act(dy, "colwise")
    dw = torch.full((128, 256), 7.0, dtype=torch.float32, device="cuda")
    fp8.gemm_wgrad(dyq, xq, out=dw, accumulate=True)
    torch.cuda.synchronize()
    assert torch.all(dw == 7.0)
    fp8.gemm_wgrad(dyq, xq, out=dw)
    torch.cuda.synchronize()
    assert torch.all(dw == 0)


def test_wgrad_f32_strided_accumulate(fp8, oracle_mod):
    """Accumulating into a column slice of a wider buffer leaves the rest alone."""
    x, dy = _operands(200, 256, 256, 53)
    xq, dyq = _quant(fp8, x, dy)
    buf = torch.full((256, 640), -3.0, dtype=torch.float32, device="cuda")
    fp8.gemm_wgrad(dyq, xq, out=buf[:, 128:384], accumulate=True)
    torch.cuda.synchronize()
    assert torch.all(buf[:, :128] == -3.0) and torch.all(buf[:, 384:] == -3.0)
    init = np.full((256, 256), -3.0)
    _check(buf[:, 128:384], oracle_mod.linear_wgrad(dy, x), init, "strided +=")


def test_linear_backward_main_grad(fp8, oracle_mod):
    x, dy = _operands(384, 256, 512, 61)
    g = torch.Generator().manual_seed(62)
    w = (torch.randn(256, 512, generator=g) * 0.02).to(torch.bfloat16)
    _, xq, wq = fp8.linear_forward(x.cuda(), w.cuda())
    main = torch.zeros(256, 512, dtype=torch.float32, device="cuda")
    for _ in range(3):
        _, dw = fp8.linear_backward(dy.cuda(), xq, wq, main_grad=main)
        assert dw is main
    torch.cuda.synchronize()
    _check(main, 3 * oracle_mod.linear_wgrad(dy, x), what="3 micro-batches")
