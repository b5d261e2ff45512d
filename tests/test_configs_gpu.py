"""Parity at the full workload sizes, in the launch configuration bench.py
times: quantizers bit-exact over the whole tensors, GEMMs within tolerance on
sampled output rows.

Workloads (fp8_block_scaled_13_b200/inputs.py): attention projections
(M=8192, QKV 2048->3072, O 2048->2048), SwiGLU gate+up (M=16384,
2048->12288, 8 channels x50), MLP down-projection with heavy tails
(M=16384, 6144->2048, Student-t(3) activations, Laplace gradients, zero
groups), and the full hidden-2048/FFN-6144 block at M = 4096, 8000 (ragged),
16384 and 32768 tokens.
"""
import numpy as np
import pytest
import torch

from helpers import assert_f32_close, assert_gemm_close, np_u8, unblock

pytestmark = pytest.mark.gpu

N_ROWS = 24  # sampled output rows per GEMM


@pytest.fixture(scope="module")
def fp8():
    import fp8_block_scaled_13_b200 as m
    from fp8_block_scaled_13_b200 import build
    build.build()
    return m


def _workload(name):
    from fp8_block_scaled_13_b200 import inputs
    if name.startswith("full_block_m"):
        return inputs.full_block(seed=4, m=int(name[len("full_block_m"):]))
    return inputs.WORKLOADS[name]()


def _sample(total, n, seed):
    rng = np.random.default_rng(seed)
    rows = rng.choice(total, size=min(n, total), replace=False)
    rows[-1] = total - 1  # always include the last (possibly ragged) row
    return np.unique(rows).astype(np.int64)


def _check_layer(fp8, oracle_mod, L, seed):
    dev = torch.device("cuda")
    x, w, dy = L.x.to(dev), L.w.to(dev), L.dy.to(dev)
    y, xq, wq = fp8.linear_forward(x, w)
    dyq = fp8.quant_act(dy, "both")
    dx = fp8.gemm_dgrad(dyq, wq)
    dw = fp8.gemm_wgrad(dyq, xq)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    m, n, k = L.m, L.n, L.k

    # ---- quantizers, whole tensors: the weight (codes, compact scales,
    # transpose, both expanded scale copies) and both activations in both
    # layouts (codes, scale bytes, zero padding of the transposed rows)
    oq, os_ = oracle_mod.quant_weight(L.w)
    assert np.array_equal(np_u8(wq.s), os_) and np.array_equal(np_u8(wq.q), oq)
    assert np.array_equal(np_u8(wq.qt), oq.T)
    assert np.array_equal(unblock(wq.s_fwd, n, k // 128), np.repeat(os_, 128, axis=0))
    assert np.array_equal(unblock(wq.s_bwd, k, n // 128), np.repeat(os_.T, 128, axis=0))
    del oq, os_
    nb = (m + 127) // 128
    for what, src, q in (("X", L.x, xq), ("dY", L.dy, dyq)):
        cols = src.shape[1]
        oq, os_ = oracle_mod.quant_rowwise(src)
        assert np.array_equal(unblock(q.s, m, cols // 128), os_), "%s %s row scales" % (L.name, what)
        assert np.array_equal(np_u8(q.q), oq), "%s %s row codes" % (L.name, what)
        del oq, os_
        oqt, ost = oracle_mod.quant_colwise(src)
        qt_full = np_u8(q.qt)
        st = unblock(q.st, cols, nb)
        assert np.array_equal(st, ost), "%s %s column scales" % (L.name, what)
        assert np.array_equal(qt_full[:, :m], oqt), "%s %s column codes" % (L.name, what)
        assert not qt_full[:, m:(m + 15) // 16 * 16].any(), "%s %s padding" % (L.name, what)
        # every all-zero 128-token band: the zero-amax scale byte and zero codes
        zero_bands = [b for b in range(nb) if not src[b * 128:(b + 1) * 128].view(torch.int16).any()]
        for b in zero_bands:
            assert (st[:, b] == 127).all()
            assert (qt_full[:, b * 128:min(m, b * 128 + 128)] == 0).all()
        del oqt, ost, qt_full, st

    # ---- GEMMs on sampled output rows
    rows = _sample(m, N_ROWS, seed + 1)
    ref = oracle_mod.linear_fprop(L.x[rows], L.w)
    assert_gemm_close(y[rows.tolist()], ref, oracle_mod, "%s fprop" % L.name)
    ref = oracle_mod.linear_dgrad(L.dy[rows], L.w)
    assert_gemm_close(dx[rows.tolist()], ref, oracle_mod, "%s dgrad" % L.name)
    cols = _sample(n, N_ROWS, seed + 2)
    ref = oracle_mod.linear_wgrad(L.dy[:, cols].contiguous(), L.x)
    assert_gemm_close(dw[cols.tolist()], ref, oracle_mod, "%s wgrad" % L.name)
    # both backward GEMMs in one launch: bit-identical to the separate calls
    dx2, dw2 = fp8.gemm_dgrad_wgrad(dyq, wq, xq)
    torch.cuda.synchronize()
    assert torch.equal(dx2.view(torch.int16), dx.view(torch.int16))
    assert torch.equal(dw2.view(torch.int16), dw.view(torch.int16))
    del dx2, dw2
    # the FP32 gradient buffer path: accumulate into an initialised buffer
    init = torch.full((n, k), 0.25, dtype=torch.float32, device=dev)
    fp8.gemm_wgrad(dyq, xq, out=init, accumulate=True)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    assert_f32_close(init[cols.tolist()], ref, np.full(ref.shape, 0.25), "%s wgrad += FP32" % L.name)


@pytest.mark.parametrize("name", ["single_fprop"])
def test_single_fprop_full(fp8, oracle_mod, name):
    L = _workload(name).layers[0]
    y, xq, wq = fp8.linear_forward(L.x.cuda(), L.w.cuda())
    torch.cuda.synchronize()
    assert_gemm_close(y, oracle_mod.linear_fprop(L.x, L.w), oracle_mod, "single fprop")
    q, s = oracle_mod.quant_rowwise(L.x)
    assert np.array_equal(np_u8(xq.q), q) and np.array_equal(unblock(xq.s, L.m, L.k // 128), s)


@pytest.mark.parametrize("name", ["attn_proj", "swiglu_gate_up", "mlp_down_heavy",
                                  "full_block_m4096", "full_block_m8000", "full_block_m16384",
                                  "full_block_m32768"])
def test_workload(fp8, oracle_mod, name):
    wl = _workload(name)
    for i, L in enumerate(wl.layers):
        _check_layer(fp8, oracle_mod, L, seed=17 * i + len(name))
        torch.cuda.empty_cache()


def test_mlp_down_heavy_has_zero_bands():
    """The heavy-tailed workload holds the zero 128-token bands that the
    column-wise zero-amax checks above run over, in X and in dY."""
    L = _workload("mlp_down_heavy").layers[0]
    for src in (L.x, L.dy):
        nb = src.shape[0] // 128
        zero = [b for b in range(nb) if not src[b * 128:(b + 1) * 128].view(torch.int16).any()]
        assert len(zero) == 8
