"""The quantizer entry point that allocates nothing.

puro_fp8_quant_act_static_scratch serves callers that own no device memory
besides their inputs and outputs (an engine whose memory pool holds the GPU's
memory, a C caller given only its buffers): the tile counter that
puro_fp8_quant_act takes from the caller lives in the library's own static
device array instead.  Its results must be those of puro_fp8_quant_act, on two
calls in a row (the second finds the array as the first left it), on a long
input that hands its tiles out by ticket and on a short one.  The test
allocates its own inputs and outputs; the entry point allocates nothing.
This file runs last so that, should it fail, every other test has run.
"""
import numpy as np
import pytest
import torch

from helpers import gpu_colwise, gpu_rowwise, np_u8

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_block_scaled_13_b200 as m
    from fp8_block_scaled_13_b200 import build
    build.build()
    return m


def _rand(shape, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * torch.exp2(torch.randint(-12, 12, shape, generator=g).float())
    return x.to(torch.bfloat16).cuda()


def _bytes(xq):
    torch.cuda.synchronize()
    q, s = gpu_rowwise(xq)
    qt, st, pad = gpu_colwise(xq)
    return q.copy(), s.copy(), qt.copy(), st.copy(), pad.copy()


def _static_scratch_call(fp8, x, xq):
    from fp8_block_scaled_13_b200 import _lib
    lib = _lib.load()
    rows, cols = x.shape
    return lib.puro_fp8_quant_act_static_scratch(
        x.data_ptr(), rows, cols, x.stride(0), _lib.PURO_BOTH, xq.q.data_ptr(), xq.q.stride(0),
        xq.s.data_ptr(), xq.qt.data_ptr(), xq.qt.stride(0), xq.st.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("rows,cols", [(40000, 1024), (300, 384)])
def test_static_scratch_matches_quant_act(fp8, rows, cols):
    x = _rand((rows, cols), rows + cols)
    ref = _bytes(fp8.quant_act(x, "both"))          # the existing entry point
    out = fp8.quant_act(x, "both")                  # buffers for the new one
    for call in range(2):
        for t in (out.q, out.qt):
            t.fill_(0x5A)
        for t in (out.s, out.st):
            t.zero_()
        assert _static_scratch_call(fp8, x, out) == 0, "call %d rejected" % call
        got = _bytes(out)
        assert fp8.device_status() == 0
        for name, a, b in zip(("q", "s", "qt", "st", "qt padding"), ref, got):
            assert np.array_equal(a, b), "call %d: %s differs from puro_fp8_quant_act" % (call, name)
