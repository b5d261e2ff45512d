"""GPU fprop/dgrad/wgrad vs the FP64 oracle.

Tolerance (block-scaled FP8 linear layer spec): relative Frobenius error
<= 1e-3 against the oracle's result rounded to BF16, and every element within
4e-3 * rms(Y_ref) + 1 BF16 ulp(Y_ref) of the unrounded FP64 result.
"""
import numpy as np
import pytest
import torch

from helpers import assert_gemm_close, gpu_colwise, gpu_rowwise

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_block_scaled_13_b200 as m
    from fp8_block_scaled_13_b200 import build
    build.build()
    return m


def _layer(m, n, k, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(m, k, generator=g).to(torch.bfloat16)
    w = (torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16)
    dy = (torch.randn(m, n, generator=g) * 1e-3).to(torch.bfloat16)
    return x, w, dy


def _run(fp8, x, w, dy):
    dev = torch.device("cuda")
    y, xq, wq = fp8.linear_forward(x.to(dev), w.to(dev))
    dx, dw = fp8.linear_backward(dy.to(dev), xq, wq)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    return y, dx, dw


@pytest.mark.parametrize("m,n,k", [
    (256, 384, 512),     # the single-fprop workload's shape
    (300, 384, 512),     # ragged token count
    (1, 128, 128),       # degenerate: one token, one block
    (129, 256, 384),
    (520, 640, 256),     # N not a multiple of the 256-wide tile
    (64, 128, 1024),
    (1300, 768, 640),    # several tiles both ways, tiles walked along N (A is larger)
    (300, 1280, 768),    # several tiles both ways, tiles walked along M (B is larger)
])
def test_linear_layer_small(fp8, oracle_mod, m, n, k):
    x, w, dy = _layer(m, n, k, m + n + k)
    y, dx, dw = _run(fp8, x, w, dy)
    assert_gemm_close(y, oracle_mod.linear_fprop(x, w), oracle_mod, "fprop")
    assert_gemm_close(dx, oracle_mod.linear_dgrad(dy, w), oracle_mod, "dgrad")
    assert_gemm_close(dw, oracle_mod.linear_wgrad(dy, x), oracle_mod, "wgrad")


def test_identity_weight_exact(fp8, oracle_mod):
    """W = I: Y equals the dequantized X exactly (each product has <= 4
    significant bits, so FP32 accumulation and BF16 rounding are exact)."""
    g = torch.Generator().manual_seed(5)
    x = (torch.randn(200, 256, generator=g) * 3).to(torch.bfloat16)
    w = torch.eye(256, dtype=torch.bfloat16)
    y, xq, wq = fp8.linear_forward(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    ref = oracle_mod.linear_fprop(x, w)
    got = y.float().cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref)
    # dgrad with W = I is exact as well
    dx = fp8.gemm_dgrad(fp8.quant_act(x.cuda(), "rowwise"), wq)
    torch.cuda.synchronize()
    assert np.array_equal(dx.float().cpu().numpy().astype(np.float64), ref)


def test_permutation_and_power_of_two_exact(fp8, oracle_mod):
    """A permutation weight and power-of-two activations: exact results."""
    g = torch.Generator().manual_seed(6)
    perm = torch.randperm(384, generator=g)
    w = torch.zeros(384, 384)
    w[torch.arange(384), perm] = 1.0
    x = torch.exp2(torch.randint(-6, 6, (130, 384), generator=g).float()) * \
        torch.where(torch.rand(130, 384, generator=g) < 0.5, -1.0, 1.0)
    x, w = x.to(torch.bfloat16), w.to(torch.bfloat16)
    y, _, _ = fp8.linear_forward(x.cuda(), w.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(y.float().cpu().numpy().astype(np.float64), oracle_mod.linear_fprop(x, w))


def test_all_ones_closed_form(fp8):
    x = torch.ones(70, 512, dtype=torch.bfloat16, device="cuda")
    w = torch.ones(256, 512, dtype=torch.bfloat16, device="cuda")
    y, _, _ = fp8.linear_forward(x, w)
    torch.cuda.synchronize()
    assert torch.all(y == 512.0)


def test_zero_tokens_wgrad_is_zero(fp8):
    x = torch.zeros(0, 256, dtype=torch.bfloat16, device="cuda")
    dy = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    xq = fp8.quant_act(x, "both")
    dyq = fp8.quant_act(dy, "both")
    dw = torch.full((128, 256), 7.0, dtype=torch.bfloat16, device="cuda")
    fp8.gemm_wgrad(dyq, xq, out=dw)
    torch.cuda.synchronize()
    assert torch.all(dw == 0)


def test_output_strides(fp8, oracle_mod):
    """Outputs written into a column slice of a wider buffer leave the rest alone."""
    x, w, _ = _layer(136, 256, 256, 9)
    xq = fp8.quant_act(x.cuda(), "rowwise")
    wq = fp8.quant_weight(w.cuda())
    buf = torch.full((136, 512), -1.0, dtype=torch.bfloat16, device="cuda")
    fp8.gemm_fprop(xq, wq, out=buf[:, 128:384])
    torch.cuda.synchronize()
    assert torch.all(buf[:, :128] == -1) and torch.all(buf[:, 384:] == -1)
    assert_gemm_close(buf[:, 128:384], oracle_mod.linear_fprop(x, w), oracle_mod, "strided fprop")


@pytest.mark.parametrize("m,n,k", [
    (300, 384, 512),      # ragged tokens
    (129, 256, 384),
    (1000, 640, 768),     # tile counts and K differ between the two products
    (128, 16384, 128),    # dgrad tiles exceed the schedule table: round-robin fallback
])
@pytest.mark.parametrize("kind", ["bf16", "f32", "f32_accumulate"])
def test_dgrad_wgrad_launch_matches_separate_calls(fp8, m, n, k, kind):
    """One launch for both backward GEMMs computes every element exactly as
    the separate calls do (only the tile-to-SM assignment differs)."""
    x, w, dy = _layer(m, n, k, 3 * m + n)
    dev = torch.device("cuda")
    xq = fp8.quant_act(x.to(dev), "colwise")
    wq = fp8.quant_weight(w.to(dev), transpose=True)
    dyq = fp8.quant_act(dy.to(dev), "both")
    dx_ref = fp8.gemm_dgrad(dyq, wq)
    if kind == "bf16":
        dw_ref = fp8.gemm_wgrad(dyq, xq)
        dx, dw = fp8.gemm_dgrad_wgrad(dyq, wq, xq)
    else:
        init = torch.randn(n, k, generator=torch.Generator().manual_seed(9)).to(dev)
        acc = kind == "f32_accumulate"
        dw_ref = fp8.gemm_wgrad(dyq, xq, out=init.clone(), accumulate=acc)
        dx, dw = fp8.gemm_dgrad_wgrad(dyq, wq, xq, dw=init.clone(), accumulate=acc)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    assert torch.equal(dx.view(torch.int16), dx_ref.view(torch.int16))
    assert torch.equal(dw.view(torch.int16 if kind == "bf16" else torch.int32),
                       dw_ref.view(torch.int16 if kind == "bf16" else torch.int32))


def test_half_width_tail_tiles_match_whole_tiles(fp8, oracle_mod):
    """A launch whose last wave would fill at most half the clusters splits
    those tiles into two half-width tiles.  Every output element is still one
    K loop in the same order: the split result equals, bit for bit, the same
    rows computed in a launch that does not split (more rows, full waves)."""
    clusters = torch.cuda.get_device_properties(0).multi_processor_count // 2
    n, k = 512, 384
    m_split = 256 * ((clusters + 1) // 2 + 1)     # 2 * tiles_m tiles -> one full wave + a few
    m_full = 256 * clusters                         # 2 * clusters tiles: whole waves, no split
    g = torch.Generator().manual_seed(77)
    x = torch.randn(m_full, k, generator=g).to(torch.bfloat16)
    w = (torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16)
    dev = torch.device("cuda")
    wq = fp8.quant_weight(w.to(dev))
    y_full = fp8.gemm_fprop(fp8.quant_act(x.to(dev), "rowwise"), wq)
    y_split = fp8.gemm_fprop(fp8.quant_act(x[:m_split].to(dev), "rowwise"), wq)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    assert torch.equal(y_split.view(torch.int16), y_full[:m_split].view(torch.int16))
    rows = np.unique(np.linspace(0, m_split - 1, 24).astype(np.int64))
    assert_gemm_close(y_split[rows.tolist()], oracle_mod.linear_fprop(x[rows], w), oracle_mod,
                      "split-tail fprop")


def test_wrapper_rejects_missing_layouts_and_bad_buffers(fp8):
    """The torch-facing wrappers refuse, before any launch, a quantization
    that lacks the layout an operation reads and an output buffer of the
    wrong shape or type."""
    x, w, dy = _layer(256, 256, 384, 21)
    dev = torch.device("cuda")
    x, w, dy = x.to(dev), w.to(dev), dy.to(dev)
    x_row = fp8.quant_act(x, "rowwise")
    x_col = fp8.quant_act(x, "colwise")
    dy_row = fp8.quant_act(dy, "rowwise")
    dy_both = fp8.quant_act(dy, "both")
    wq = fp8.quant_weight(w)
    wq_fwd = fp8.quant_weight(w, transpose=False)
    with pytest.raises(ValueError):
        fp8.gemm_fprop(x_col, wq)                               # no row-wise codes
    with pytest.raises(ValueError):
        fp8.gemm_fprop(x_row, wq, out=torch.empty(256, 128, dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError):
        fp8.gemm_fprop(x_row, wq, out=torch.empty(256, 256, dtype=torch.float32, device=dev))
    with pytest.raises(ValueError):
        fp8.gemm_dgrad(dy_row, wq_fwd)                          # no transposed weight
    with pytest.raises(ValueError):
        fp8.gemm_dgrad(dy_row, wq, out=torch.empty(255, 384, dtype=torch.bfloat16, device=dev))
    with pytest.raises(ValueError):
        fp8.gemm_wgrad(dy_row, x_col)                           # dY lacks column-wise codes
    with pytest.raises(ValueError):
        fp8.gemm_wgrad(dy_both, x_col, out=torch.empty(384, 256, dtype=torch.float32, device=dev))
    with pytest.raises(ValueError):
        fp8.gemm_wgrad(dy_both, x_col, out=torch.empty(256, 384, dtype=torch.bfloat16, device=dev),
                       accumulate=True)
    with pytest.raises(ValueError):
        fp8.gemm_dgrad_wgrad(dy_both, wq, x_row)                # X lacks column-wise codes
    with pytest.raises(ValueError):
        fp8.gemm_dgrad_wgrad(dy_both, wq, x_col, dx=torch.empty(256, 384, dtype=torch.float32, device=dev))
    with pytest.raises(ValueError):
        fp8.quant_act(x, "both", out=x_row)                     # reused result lacks the transposed layout
    with pytest.raises(ValueError):
        fp8.quant_act(x[:128].contiguous(), "rowwise", out=x_row)   # made for another shape
    with pytest.raises(ValueError):
        fp8.quant_weight(w[:128].contiguous(), out=wq)
    with pytest.raises(ValueError, match="layout"):
        fp8.quant_act(x, "row")                                 # unknown layout name
    # reusing a matching result works and gives the same codes
    again = fp8.quant_act(x, "rowwise", out=fp8.QuantAct(256, 384, torch.empty_like(x_row.q),
                                                          torch.empty_like(x_row.s)))
    torch.cuda.synchronize()
    assert torch.equal(again.q, x_row.q)
    # only the scales of real groups are defined: bytes of the fourth (absent)
    # group slot are left as they were
    assert np.array_equal(gpu_rowwise(again)[1], gpu_rowwise(x_row)[1])
    assert fp8.device_status() == 0


def test_wrapper_rejects_short_scale_buffers(fp8):
    """A QuantAct or QuantWeight whose scale buffers are smaller than their
    blocked layout (a caller-built or reused result) is refused before the
    launch: the kernel's tensor maps would read past the buffers' ends."""
    import dataclasses
    x, w, dy = _layer(256, 256, 384, 22)
    dev = torch.device("cuda")
    x, w, dy = x.to(dev), w.to(dev), dy.to(dev)
    xq = fp8.quant_act(x, "both")
    dyq = fp8.quant_act(dy, "both")
    wq = fp8.quant_weight(w)
    short = lambda t: t[: t.numel() - 16]
    with pytest.raises(ValueError, match="bytes"):
        fp8.gemm_fprop(dataclasses.replace(xq, s=short(xq.s)), wq)
    with pytest.raises(ValueError, match="bytes"):
        fp8.gemm_fprop(xq, dataclasses.replace(wq, s_fwd=short(wq.s_fwd)))
    with pytest.raises(ValueError, match="bytes"):
        fp8.gemm_dgrad(dyq, dataclasses.replace(wq, s_bwd=short(wq.s_bwd)))
    with pytest.raises(ValueError, match="bytes"):
        fp8.gemm_wgrad(dataclasses.replace(dyq, st=short(dyq.st)), xq)
    with pytest.raises(ValueError, match="bytes"):
        fp8.gemm_dgrad_wgrad(dyq, wq, dataclasses.replace(xq, st=short(xq.st)))
    with pytest.raises(ValueError):
        fp8.gemm_fprop(dataclasses.replace(xq, q=xq.q[:, :256]), wq)    # codes narrower than K
    assert fp8.device_status() == 0


def test_wrappers_launch_on_the_current_stream(fp8):
    """The wrappers hand the library the caller's current stream: the default
    stream, or the one a `torch.cuda.stream` context makes current.  A layer
    run on a side stream equals the same layer on the default stream."""
    from fp8_block_scaled_13_b200 import linear
    assert linear._stream() == torch.cuda.current_stream().cuda_stream
    x, w, dy = _layer(300, 256, 384, 31)
    want = _run(fp8, x, w, dy)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        assert linear._stream() == s.cuda_stream
        dev = torch.device("cuda")
        xd, wd, dyd = x.to(dev), w.to(dev), dy.to(dev)
        y, xq, wq = fp8.linear_forward(xd, wd)
        dx, dw = fp8.linear_backward(dyd, xq, wq)
    s.synchronize()
    for a, b in zip((y, dx, dw), want):
        assert torch.equal(a, b)
