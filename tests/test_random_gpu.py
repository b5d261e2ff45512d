"""Randomized parity: hypothesis draws shapes, row strides, layouts and value
ranges, and every draw is compared with the oracle -- the quantizers bit for
bit over the whole tensor, the linear layer's three GEMMs within the spec's
tolerance.  Draws are derandomized, so a failure reproduces."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings, strategies as st

from helpers import assert_gemm_close, gpu_colwise, gpu_rowwise

pytestmark = pytest.mark.gpu

SETTINGS = dict(deadline=None, derandomize=True, suppress_health_check=list(HealthCheck))


@pytest.fixture(scope="module")
def fp8():
    import fp8_block_scaled_13_b200 as m
    from fp8_block_scaled_13_b200 import build
    build.build()
    return m


def _values(rows, cols, seed, spread):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(rows, cols, generator=g)
    if spread:
        x = x * torch.exp2(torch.randint(-spread, spread + 1, (rows, cols), generator=g).float())
    return x.to(torch.bfloat16)


@settings(max_examples=40, **SETTINGS)
@given(rows=st.integers(1, 2600), ncol=st.integers(1, 12), pad=st.sampled_from([0, 8, 136]),
       layout=st.sampled_from(["rowwise", "colwise", "both"]), spread=st.sampled_from([0, 6, 30]),
       seed=st.integers(0, 2 ** 31 - 1))
def test_quant_act_random(fp8, oracle_mod, rows, ncol, pad, layout, spread, seed):
    cols = 128 * ncol
    x = _values(rows, cols, seed, spread)
    full = torch.zeros(rows, cols + pad, dtype=torch.bfloat16, device="cuda")
    full[:, :cols] = x.cuda()
    xq = fp8.quant_act(full[:, :cols], layout)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    if xq.q is not None:
        q, s = gpu_rowwise(xq)
        oq, os_ = oracle_mod.quant_rowwise(x)
        assert np.array_equal(s, os_) and np.array_equal(q, oq), "rowwise differs"
    if xq.qt is not None:
        qt, stt, padb = gpu_colwise(xq)
        oqt, ost = oracle_mod.quant_colwise(x)
        assert np.array_equal(stt, ost) and np.array_equal(qt, oqt), "colwise differs"
        assert not padb.any()
    if xq.work is not None:
        assert not xq.work.any(), "tile counter not reset"


@settings(max_examples=20, **SETTINGS)
@given(m=st.integers(1, 1500), nb=st.integers(1, 10), kb=st.integers(1, 8), seed=st.integers(0, 2 ** 31 - 1))
def test_linear_layer_random(fp8, oracle_mod, m, nb, kb, seed):
    n, k = 128 * nb, 128 * kb
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(m, k, generator=g).to(torch.bfloat16)
    w = (torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16)
    dy = (torch.randn(m, n, generator=g) * 1e-3).to(torch.bfloat16)
    dev = torch.device("cuda")
    y, xq, wq = fp8.linear_forward(x.to(dev), w.to(dev))
    dx, dw = fp8.linear_backward(dy.to(dev), xq, wq)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    assert_gemm_close(y, oracle_mod.linear_fprop(x, w), oracle_mod, "fprop")
    assert_gemm_close(dx, oracle_mod.linear_dgrad(dy, w), oracle_mod, "dgrad")
    assert_gemm_close(dw, oracle_mod.linear_wgrad(dy, x), oracle_mod, "wgrad")


@settings(max_examples=8, **SETTINGS)
@given(rows=st.integers(20000, 45000), ncol=st.integers(8, 12), pad=st.sampled_from([0, 8]),
       layout=st.sampled_from(["rowwise", "colwise", "both"]), seed=st.integers(0, 2 ** 31 - 1))
def test_quant_act_random_long(fp8, oracle_mod, rows, ncol, pad, layout, seed):
    """Long inputs (past 16 tiles per SM on a B200, so the tiles go out by
    ticket), ragged row counts, strided rows."""
    cols = 128 * ncol
    x = _values(rows, cols, seed, 8)
    full = torch.zeros(rows, cols + pad, dtype=torch.bfloat16, device="cuda")
    full[:, :cols] = x.cuda()
    xq = fp8.quant_act(full[:, :cols], layout)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    if xq.q is not None:
        q, s = gpu_rowwise(xq)
        oq, os_ = oracle_mod.quant_rowwise(x)
        assert np.array_equal(s, os_) and np.array_equal(q, oq), "rowwise differs"
    if xq.qt is not None:
        qt, stt, padb = gpu_colwise(xq)
        oqt, ost = oracle_mod.quant_colwise(x)
        assert np.array_equal(stt, ost) and np.array_equal(qt, oqt), "colwise differs"
        assert not padb.any()
    assert not xq.work.any(), "tile counter not reset"
