"""GPU quantizers vs the CPU oracle: codes and scale bytes must match bit for bit."""
import numpy as np
import pytest
import torch

from helpers import blocked_index, gpu_colwise, gpu_rowwise, np_u8, unblock

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fp8():
    import fp8_block_scaled_13_b200 as m
    from fp8_block_scaled_13_b200 import build
    build.build()
    return m


def _rand(shape, seed, lo=-20, hi=20):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * torch.exp2(
        torch.randint(lo, hi, shape, generator=g).float())
    return x.to(torch.bfloat16)


def _check_all(fp8, oracle_mod, x, layout="both"):
    xq = fp8.quant_act(x.cuda(), layout)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    if xq.q is not None:
        q, s = gpu_rowwise(xq)
        oq, os_ = oracle_mod.quant_rowwise(x)
        assert np.array_equal(s, os_), "rowwise scales differ"
        assert np.array_equal(q, oq), "rowwise codes differ at %s" % (np.argwhere(q != oq)[:5],)
    if xq.qt is not None:
        qt, st, pad = gpu_colwise(xq)
        oqt, ost = oracle_mod.quant_colwise(x)
        assert np.array_equal(st, ost), "colwise scales differ"
        assert np.array_equal(qt, oqt), "colwise codes differ at %s" % (np.argwhere(qt != oqt)[:5],)
        assert not pad.any(), "padding of the transposed codes is not zero"
    return xq


@pytest.mark.parametrize("rows,cols", [(1, 128), (300, 384), (128, 1024), (257, 256), (1000, 640)])
@pytest.mark.parametrize("layout", ["rowwise", "colwise", "both"])
def test_quant_act_random(fp8, oracle_mod, rows, cols, layout):
    _check_all(fp8, oracle_mod, _rand((rows, cols), rows * 7 + cols), layout)


def test_quant_act_every_bf16_pattern(fp8, oracle_mod):
    """Every finite BF16 value appears once as an element (510 rows x 128)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    bits = bits[((bits >> 7) & 0xFF) != 0xFF]
    assert bits.size == 510 * 128
    rng = np.random.default_rng(0)
    rng.shuffle(bits)
    x = torch.from_numpy(bits.view(np.int16).reshape(510, 128).copy()).view(torch.bfloat16)
    _check_all(fp8, oracle_mod, x, "both")
    # and sorted, so that each group spans a narrow range of magnitudes
    xs = torch.from_numpy(np.sort(bits).view(np.int16).reshape(510, 128).copy()).view(torch.bfloat16)
    _check_all(fp8, oracle_mod, xs, "both")


def test_quant_act_adversarial_groups(fp8, oracle_mod):
    x = _rand((256, 1280), 11).float()
    x[0, 0:128] = 0.0                                  # all-zero group
    x[1, 0:128] = -0.0                                 # negative zeros
    x[2, 0:128] = torch.linspace(-1, 1, 128) * 2.0 ** -130   # subnormal-only
    x[3, 0:128] = 1e-3
    x[3, 5] = 448.0                                    # amax exactly 448
    x[4, 0:128] = 1e-3
    x[4, 9] = -450.0                                   # next BF16 above 448
    for kk, k in enumerate(range(-10, 10, 4)):
        x[5 + kk, 128:256] = 0.5
        x[5 + kk, 130] = 448.0 * 2.0 ** k              # amax = 448 * 2^k
        x[5 + kk, 256:384] = 0.5
        x[5 + kk, 300] = 450.0 * 2.0 ** k              # just above it
    x[20, 384:512] = 1.0
    x[20, 400] = 3.0e38                                # near BF16 max
    x[21, 512:640] = torch.arange(128) * 2.0 ** -133   # smallest subnormals
    x[22:150, 640:768] = 0.0                           # zero rows straddling two 128-row groups
    x[128:256, 1152:1280] = 0.0                        # an aligned zero 128-row group in 128 columns
    x[128:256, 1100] = -0.0                            # a column group of negative zeros
    x[30, 768:896] = 224.0                             # half of 448: exponent boundary
    x[31, 768:896] = 1.75                              # 1.75 = 448 * 2^-8
    x[32, 768:896] = 1.78125
    xq = _check_all(fp8, oracle_mod, x.to(torch.bfloat16), "both")
    # the zero-amax path of the column-wise quantizer, byte by byte: scale
    # byte 127 (e = 0) and codes 0x00 (or 0x80 for -0) in the zero groups
    qt, st, _ = gpu_colwise(xq)
    assert (st[1152:1280, 1] == 127).all()
    assert (qt[1152:1280, 128:256] == 0).all()
    assert st[1100, 1] == 127 and (qt[1100, 128:256] == 0x80).all()
    # and the row-wise zero groups
    q, s = gpu_rowwise(xq)
    assert s[0, 0] == 127 and (q[0, 0:128] == 0).all()
    assert s[1, 0] == 127 and (q[1, 0:128] == 0x80).all()


def test_quant_act_zero_ragged_column_group(fp8, oracle_mod):
    """A short last token group (300 rows: 44 in the third group) that is all
    zero in some columns, and an aligned full zero group, in every layout."""
    x = _rand((300, 384), 21).float()
    x[256:300, 0:64] = 0.0         # the short last group of columns 0..63
    x[128:256, 128:256] = 0.0      # a full 128-row group of columns 128..255
    for layout in ("colwise", "both"):
        xq = _check_all(fp8, oracle_mod, x.to(torch.bfloat16), layout)
        qt, st, pad = gpu_colwise(xq)
        assert (st[0:64, 2] == 127).all() and (qt[0:64, 256:300] == 0).all()
        assert (st[128:256, 1] == 127).all() and (qt[128:256, 128:256] == 0).all()
        assert (st[64:, 2] != 127).any()   # the other columns' last groups are not zero


def test_quant_act_strided_input(fp8, oracle_mod):
    """A column slice of a wider tensor (ld_x > cols) and rows not multiple of 16."""
    base = _rand((200, 768), 12)
    xv = base.cuda()[:, 128:512]
    assert xv.stride(0) == 768
    xq = fp8.quant_act(xv, "both")
    torch.cuda.synchronize()
    x = base[:, 128:512].contiguous()
    q, s = gpu_rowwise(xq)
    oq, os_ = oracle_mod.quant_rowwise(x)
    assert np.array_equal(q, oq) and np.array_equal(s, os_)
    qt, st, pad = gpu_colwise(xq)
    oqt, ost = oracle_mod.quant_colwise(x)
    assert np.array_equal(qt, oqt) and np.array_equal(st, ost) and not pad.any()


@pytest.mark.parametrize("n,k", [(128, 128), (384, 512), (3072, 2048), (2048, 6144)])
def test_quant_weight(fp8, oracle_mod, n, k):
    g = torch.Generator().manual_seed(n + k)
    w = (torch.randn(n, k, generator=g) * 0.02).to(torch.bfloat16)
    w[:128, :128] = 0   # a zero block
    wq = fp8.quant_weight(w.cuda(), transpose=True)
    torch.cuda.synchronize()
    oq, os_ = oracle_mod.quant_weight(w)
    assert np.array_equal(np_u8(wq.s), os_)
    assert np.array_equal(np_u8(wq.q), oq)
    assert np.array_equal(np_u8(wq.qt), oq.T)
    # expanded per-row copies in the GEMM's blocked layout
    fwd = unblock(wq.s_fwd, n, k // 128)
    bwd = unblock(wq.s_bwd, k, n // 128)
    assert np.array_equal(fwd, np.repeat(os_, 128, axis=0))
    assert np.array_equal(bwd, np.repeat(os_.T, 128, axis=0))


def test_quant_weight_heavy_tails(fp8, oracle_mod):
    w = _rand((256, 384), 13, -30, 30)
    wq = fp8.quant_weight(w.cuda(), transpose=False)
    torch.cuda.synchronize()
    oq, os_ = oracle_mod.quant_weight(w)
    assert np.array_equal(np_u8(wq.s), os_) and np.array_equal(np_u8(wq.q), oq)
    assert wq.qt is None and wq.s_bwd is None
    assert np.array_equal(unblock(wq.s_fwd, 256, 3), np.repeat(os_, 128, axis=0))


def test_bounded_wait_reports_timeout(fp8):
    """A wait that can never complete gives up, records the timeout and returns."""
    from fp8_block_scaled_13_b200 import _lib
    assert fp8.device_status() == 0
    st = _lib.puro_fp8_test_bounded_wait(20_000_000, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    assert fp8.device_status() == _lib.PURO_ERR_DEVICE_TIMEOUT
    assert fp8.device_status() == 0   # cleared by the read
    # the context is still usable
    x = _rand((128, 128), 14).cuda()
    fp8.quant_act(x, "rowwise")
    torch.cuda.synchronize()


def test_blocked_layout_padding_rows(fp8):
    """Rows past the end of the last 128-row block carry the zero-group byte 127."""
    x = _rand((200, 256), 15).cuda()
    xq = fp8.quant_act(x, "rowwise")
    torch.cuda.synchronize()
    full = unblock(xq.s, 256, 2)
    assert np.all(full[200:] == 127)


def test_blocked_index_is_a_bijection():
    idx = blocked_index(384, 8)
    assert np.unique(idx).size == idx.size and idx.max() == 3 * 2 * 512 - 1


def _outs(xq):
    """Every byte the call defines: the codes (the transposed codes with their
    zero padding columns) and the scale bytes of the existing groups (the
    padding groups of a blocked array are not written)."""
    torch.cuda.synchronize()
    out = []
    if xq.q is not None:
        q, s = gpu_rowwise(xq)
        out += [q.copy(), s.copy()]
    if xq.qt is not None:
        out += [np_u8(xq.qt).copy(), gpu_colwise(xq)[1].copy()]
    return out


def _same(a, b):
    return len(a) == len(b) and all(np.array_equal(x, y) for x, y in zip(a, b))


def _long_stream(rows, cols):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return -(-rows // 128) * (cols // 128) > 16 * sms


@pytest.mark.parametrize("rows,cols,layout", [(40000, 1024, "both"), (33001, 2048, "rowwise"),
                                              (20000, 2048, "colwise"),
                                              (300, 128 * 3001, "both"),   # 3001 column tiles
                                              (1000003, 128, "both")])     # one column tile
def test_tile_counter_long_streams(fp8, oracle_mod, rows, cols, layout):
    """Long inputs (more than 16 tiles per SM) hand their tiles out by ticket
    from the output's counter: the oracle's bytes over the whole tensor (ragged
    last row tile included), the same bytes as the static schedule, and the
    counter back at zero after every call.  The last two shapes take the tile
    decode (row tile = ticket tile / column tiles, by multiply-shift) to an odd
    divisor of 3001 and to the single-column-tile case."""
    assert _long_stream(rows, cols)
    x = _rand((rows, cols), rows + cols)
    xq = _check_all(fp8, oracle_mod, x, layout)
    assert xq.work is not None and not xq.work.any(), "tile counter not reset"
    ref = _outs(xq)
    xc = x.cuda()
    for _ in range(2):  # the same counter again: same bytes
        fp8.quant_act(xc, layout, out=xq)
        torch.cuda.synchronize()
        assert not xq.work.any(), "tile counter not reset"
        assert _same(ref, _outs(xq))
    static = fp8.quant_act(xc, layout)
    static.work = None
    for t in (static.q, static.s, static.qt, static.st):
        if t is not None:
            t.zero_()
    fp8.quant_act(xc, layout, out=static)
    torch.cuda.synchronize()
    assert fp8.device_status() == 0
    assert _same(ref, _outs(static))


def test_tile_counter_graph_replays(fp8):
    """Two ticket-scheduled launches captured in one CUDA graph on the same
    counter, replayed three times: every replay rewrites the same bytes and
    leaves the counter at zero."""
    x = _rand((40000, 1024), 9).cuda()
    xq = fp8.quant_act(x, "both")
    torch.cuda.synchronize()
    ref = _outs(xq)
    g = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        with torch.cuda.graph(g, stream=cap):
            fp8.quant_act(x, "both", out=xq)
            fp8.quant_act(x, "both", out=xq)
    torch.cuda.synchronize()
    for _ in range(3):
        for t in (xq.q, xq.s, xq.qt, xq.st):
            t.fill_(0x5A)
        g.replay()
        torch.cuda.synchronize()
        assert fp8.device_status() == 0
        assert not xq.work.any(), "tile counter not reset"
        assert _same(ref, _outs(xq))
    del g


@pytest.mark.parametrize("case", ["static_edge", "ticket_edge", "ticket_narrow3_ragged"])
def test_tile_counter_threshold(fp8, oracle_mod, case):
    """Both sides of the ticket threshold (16 tiles per SM), against the oracle
    over the whole tensor: the last static-schedule size, the first ticket
    size (one tile per row of tiles, so the tile decode is the identity), and
    a three-tile-wide ragged input just past the threshold (multiply-shift
    decode)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    limit = 16 * sms
    rows, cols = {"static_edge": (limit * 128, 128),
                  "ticket_edge": ((limit + 1) * 128, 128),
                  "ticket_narrow3_ragged": ((limit // 3 + 1) * 128 - 37, 384)}[case]
    tiles = -(-rows // 128) * (cols // 128)
    assert (tiles > limit) == (case != "static_edge")
    xq = _check_all(fp8, oracle_mod, _rand((rows, cols), tiles), "both")
    assert not xq.work.any(), "tile counter not reset"
