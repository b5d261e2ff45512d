"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each test ties one oracle function to a closed form, a brute-force search, an
exact integer restatement, a library routine that is RUN (torch's
float8_e4m3fn cast, numpy matmul), or a hand-derived worked example
(tests/golden/e4m3_worked_examples.txt).  The cases are chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand,
the wrong group size, ties rounded away from even, the floor instead of the
ceiling scale rule) fails at least one of them.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_worked_examples.txt")


def _all_bf16_finite():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    exp = (bits >> 7) & 0xFF
    return bits[exp != 0xFF]


def _positive_codes(oracle_mod):
    codes = np.arange(0x7F, dtype=np.uint8)  # 0x00 .. 0x7E, all finite non-negative
    return codes, oracle_mod.e4m3_decode(codes)


def _brute_force_encode(values, codes, vals):
    """Nearest finite E4M3 magnitude; ties go to the even code; beyond 448 the
    result saturates to 448.  Sign copied from the input."""
    v = np.asarray(values, np.float64)
    a = np.minimum(np.abs(v), 448.0)
    d = np.abs(a[:, None] - vals[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among tied candidates prefer the even code
    even = (codes[None, :] % 2) == 0
    pick_even = cand & even
    has_even = pick_even.any(axis=1)
    idx = np.where(has_even, pick_even.argmax(axis=1), cand.argmax(axis=1))
    out = codes[idx].astype(np.uint8)
    out |= np.where(np.signbit(v), 0x80, 0).astype(np.uint8)
    return out


# ---------------------------------------------------------------- golden file

def _golden():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            rows.append(line.split())
    return rows


def _parse_num(s):
    return float.fromhex(s) if "0x" in s else float(s)


def test_golden_decode(oracle_mod):
    n = 0
    for kind, a, b in _golden():
        if kind != "decode":
            continue
        got = oracle_mod.e4m3_decode(np.uint8(int(a, 16)))
        want = _parse_num(b)
        assert got == want and math.copysign(1, got) == math.copysign(1, want), (a, got, want)
        n += 1
    assert n >= 10


def test_golden_encode(oracle_mod):
    n = 0
    for kind, a, b in _golden():
        if kind != "encode":
            continue
        got = int(oracle_mod.e4m3_encode(_parse_num(a)))
        assert got == int(b, 16), (a, hex(got), b)
        n += 1
    assert n >= 10


def test_golden_scale(oracle_mod):
    n = 0
    for kind, a, b in _golden():
        if kind != "scale":
            continue
        assert oracle_mod.scale_exponent(_parse_num(a)) == int(b), a
        n += 1
    assert n >= 10


# ---------------------------------------------------------------- E4M3 codec

def test_decode_closed_form_every_code(oracle_mod):
    """Sign/exponent/mantissa fields per the 4-exponent/3-mantissa layout."""
    vals = oracle_mod.e4m3_decode(np.arange(256, dtype=np.uint8))
    for c in range(256):
        s, E, m = c >> 7, (c >> 3) & 15, c & 7
        if E == 15 and m == 7:
            assert np.isnan(vals[c])
            continue
        mag = (m / 8) * 2.0 ** -6 if E == 0 else (1 + m / 8) * 2.0 ** (E - 7)
        assert vals[c] == (-mag if s else mag)
    assert np.nanmax(vals) == 448.0 and np.nanmin(vals) == -448.0


def test_decode_matches_torch_float8(oracle_mod):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle_mod.e4m3_decode(np.arange(256, dtype=np.uint8))
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.all(both_nan | (ref == got))


def test_encode_brute_force_all_bf16(oracle_mod):
    """Every finite BF16 value: nearest-code brute force with ties to even."""
    bits = _all_bf16_finite()
    vals = oracle_mod.bf16_to_double(bits)
    codes, dec = _positive_codes(oracle_mod)
    want = np.concatenate([_brute_force_encode(vals[i:i + 8192], codes, dec)
                           for i in range(0, vals.size, 8192)])
    got = oracle_mod.e4m3_encode(vals)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(vals[i], got[i], want[i]) for i in bad[:5]]


def test_encode_midpoints_tie_to_even(oracle_mod):
    """Exact midpoints between neighbouring codes go to the even code, and a
    hair either side of a midpoint goes to the nearer code."""
    codes, dec = _positive_codes(oracle_mod)
    mids = (dec[:-1] + dec[1:]) / 2.0
    got = oracle_mod.e4m3_encode(mids)
    want = np.where(codes[:-1] % 2 == 0, codes[:-1], codes[1:])
    assert np.array_equal(got, want)
    below = oracle_mod.e4m3_encode(np.nextafter(mids, 0))
    above = oracle_mod.e4m3_encode(np.nextafter(mids, np.inf))
    assert np.array_equal(below, codes[:-1])
    assert np.array_equal(above, codes[1:])


def test_encode_matches_torch_cast(oracle_mod):
    """torch's float8_e4m3fn cast is a library RNE conversion; it agrees with
    the oracle wherever |v| <= 448 (the only range the scale rule produces)."""
    g = torch.Generator().manual_seed(123)
    v = torch.randn(200000, generator=g, dtype=torch.float64) * torch.exp2(
        torch.randint(-14, 9, (200000,), generator=g).to(torch.float64))
    v = v.clamp(-448, 448)
    ref = v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle_mod.e4m3_encode(v.numpy())
    assert np.array_equal(got, ref)


def test_encode_signed_zero_and_saturation(oracle_mod):
    assert oracle_mod.e4m3_encode(-1e-30) == 0x80
    assert oracle_mod.e4m3_encode(1e-30) == 0x00
    assert oracle_mod.e4m3_encode(1e9) == 0x7E
    assert oracle_mod.e4m3_encode(-1e9) == 0xFE


# ---------------------------------------------------------------- scale rule

def test_scale_rule_closed_form(oracle_mod):
    """e = smallest integer with amax <= 448*2^e.  With amax = f*2^p,
    f in [0.5,1): amax <= 0.875*2^(p+9+e'), so e = p-9 if f <= 0.875 else p-8,
    then clamped to [-127, 127]."""
    g = np.random.default_rng(7)
    amax = np.concatenate([
        g.random(20000) * 2.0 ** g.integers(-140, 128, 20000),
        oracle_mod.bf16_to_double(_all_bf16_finite()),
    ])
    amax = np.abs(amax)
    for a in amax[::7]:
        if a == 0:
            want = 0
        else:
            f, p = math.frexp(a)
            want = p - 9 if f <= 0.875 else p - 8
            want = max(-127, min(127, want))
        assert oracle_mod.scale_exponent(a) == want, a


def test_scale_rule_invariants(oracle_mod):
    """Power of two with amax/scale <= 448, and minimal (unless clamped)."""
    for a in oracle_mod.bf16_to_double(_all_bf16_finite())[::13]:
        a = abs(a)
        e = oracle_mod.scale_exponent(a)
        assert -127 <= e <= 127
        assert a <= 448.0 * 2.0 ** e
        if a != 0 and e > -127:
            assert a > 448.0 * 2.0 ** (e - 1)


# ---------------------------------------------------------------- quantizers

def _brute_quant_group(vals, codes, dec):
    vals = np.asarray(vals, np.float64)
    amax = np.abs(vals).max()
    if amax == 0:
        e = 0
    else:
        e = 0
        while amax > 448.0 * 2.0 ** e:
            e += 1
        while e > -127 and amax <= 448.0 * 2.0 ** (e - 1):
            e -= 1
    q = _brute_force_encode(vals * 2.0 ** -e, codes, dec)
    return q, e + 127


def _rand_bf16(shape, seed, scale_pow=(-20, 20)):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(*shape, generator=g) * torch.exp2(
        torch.randint(scale_pow[0], scale_pow[1], shape, generator=g).float())
    return x.to(torch.bfloat16)


def test_quant_rowwise_brute_force(oracle_mod):
    codes, dec = _positive_codes(oracle_mod)
    x = _rand_bf16((5, 384), 1)
    x[2, 128:256] = 0
    q, s = oracle_mod.quant_rowwise(x)
    xd = x.double().numpy()
    for r in range(5):
        for gi in range(3):
            wq, ws = _brute_quant_group(xd[r, gi * 128:(gi + 1) * 128], codes, dec)
            assert np.array_equal(q[r, gi * 128:(gi + 1) * 128], wq)
            assert s[r, gi] == ws
    assert s[2, 1] == 127 and np.all(q[2, 128:256] % 128 == 0)


def test_quant_colwise_brute_force_ragged(oracle_mod):
    """Columns grouped by 128 rows; the last group (2 rows) is short and its
    amax covers only its valid rows."""
    codes, dec = _positive_codes(oracle_mod)
    x = _rand_bf16((130, 6), 2)
    x[0, :] = 1000.0    # big values in the first group only
    qt, st = oracle_mod.quant_colwise(x)
    assert qt.shape == (6, 130) and st.shape == (6, 2)
    xd = x.double().numpy()
    for c in range(6):
        for gi, (r0, r1) in enumerate([(0, 128), (128, 130)]):
            wq, ws = _brute_quant_group(xd[r0:r1, c], codes, dec)
            assert np.array_equal(qt[c, r0:r1], wq)
            assert st[c, gi] == ws


def test_quant_colwise_is_rowwise_of_transpose(oracle_mod):
    x = _rand_bf16((256, 384), 3)
    qt, st = oracle_mod.quant_colwise(x)
    q2, s2 = oracle_mod.quant_rowwise(x.t().contiguous())
    assert np.array_equal(qt, q2) and np.array_equal(st, s2)


def test_group_size_is_128(oracle_mod):
    """Perturbing one element changes exactly the scale of its own 1x128 group
    (rowwise) or its own 128x128 block (weights)."""
    x = _rand_bf16((4, 512), 4, (0, 1))
    _, s0 = oracle_mod.quant_rowwise(x)
    x2 = x.clone()
    x2[1, 300] = 1e4
    _, s1 = oracle_mod.quant_rowwise(x2)
    diff = np.argwhere(s0 != s1)
    assert diff.tolist() == [[1, 300 // 128]]
    w = _rand_bf16((256, 384), 5, (0, 1))
    _, sw0 = oracle_mod.quant_weight(w)
    w2 = w.clone()
    w2[200, 140] = 1e4
    _, sw1 = oracle_mod.quant_weight(w2)
    assert np.argwhere(sw0 != sw1).tolist() == [[1, 1]]


def test_quant_weight_brute_force(oracle_mod):
    codes, dec = _positive_codes(oracle_mod)
    w = _rand_bf16((256, 256), 6, (-3, 3))
    q, s = oracle_mod.quant_weight(w)
    wd = w.double().numpy()
    for bn in range(2):
        for bk in range(2):
            blk = wd[bn * 128:(bn + 1) * 128, bk * 128:(bk + 1) * 128]
            wq, ws = _brute_quant_group(blk.reshape(-1), codes, dec)
            assert np.array_equal(q[bn * 128:(bn + 1) * 128, bk * 128:(bk + 1) * 128].reshape(-1), wq)
            assert s[bn, bk] == ws


def test_quant_weight_transpose_consistent(oracle_mod):
    """128x128 blocks are square: quantizing W^T gives the byte transpose of
    Qw and of the scale grid (what dgrad relies on)."""
    w = _rand_bf16((384, 256), 7)
    q, s = oracle_mod.quant_weight(w)
    qt, st = oracle_mod.quant_weight(w.t().contiguous())
    assert np.array_equal(qt, q.T) and np.array_equal(st, s.T)


def test_scaled_amax_bounds_every_group(oracle_mod):
    """amax/scale <= 448 in every group, > 224 unless the group is zero or clamped."""
    x = _rand_bf16((64, 1024), 8)
    q, s = oracle_mod.quant_rowwise(x)
    xd = x.double().numpy().reshape(64, 8, 128)
    amax = np.abs(xd).max(axis=2)
    scaled = amax * 2.0 ** -(s.astype(np.int64) - 127)
    assert np.all(scaled <= 448) and np.all(scaled > 224)


# ---------------------------------------------------------------- dequant + GEMMs

def test_dequant_exact(oracle_mod):
    g = np.random.default_rng(9)
    q = g.integers(0, 256, (3, 256), dtype=np.uint8)
    q[q % 128 == 0x7F] = 0x11
    s = g.integers(100, 150, (3, 2), dtype=np.uint8)
    d = oracle_mod.dequant_groups(q, s)
    dec = oracle_mod.e4m3_decode(np.arange(256, dtype=np.uint8))
    for r in range(3):
        for c in range(256):
            assert d[r, c] == dec[q[r, c]] * 2.0 ** (int(s[r, c // 128]) - 127)


def _exact_int(code):
    """E4M3 value as an integer multiple of 2^-9 (exact)."""
    s, E, m = code >> 7, (code >> 3) & 15, code & 7
    n = m if E == 0 else (8 + m) << (E - 1)
    return -n if s else n


def test_gemm_exact_integer_restatement(oracle_mod):
    """Each E4M3 value is an integer times 2^-9, so each 128-block dot product is
    an exact integer times 2^(ea+eb-18); summed as exact rationals this is the
    gold result.  The FP64 oracle must agree within FP64 summation error."""
    x = _rand_bf16((3, 256), 10)
    w = _rand_bf16((128, 256), 11, (-6, 6))
    qx, sx = oracle_mod.quant_rowwise(x)
    qw, sw = oracle_mod.quant_weight(w)
    y = oracle_mod.gemm_fprop(oracle_mod.dequant_groups(qx, sx),
                              oracle_mod.dequant_blocks(qw, sw))
    for m in range(3):
        for n in range(0, 128, 17):
            tot = Fraction(0)
            mag = Fraction(0)
            for kb in range(2):
                dot = sum(_exact_int(int(qx[m, k])) * _exact_int(int(qw[n, k]))
                          for k in range(kb * 128, kb * 128 + 128))
                absdot = sum(abs(_exact_int(int(qx[m, k])) * _exact_int(int(qw[n, k])))
                             for k in range(kb * 128, kb * 128 + 128))
                sc = Fraction(2) ** (int(sx[m, kb]) - 127 + int(sw[n // 128, kb]) - 127 - 18)
                tot += dot * sc
                mag += absdot * sc
            err = abs(Fraction(y[m, n]) - tot)
            assert err <= mag * Fraction(256 * 2, 2 ** 53), (m, n)


def test_gemm_matches_numpy_matmul(oracle_mod):
    """numpy's BLAS matmul on the same FP64 operands: equal up to FP64 rounding."""
    g = np.random.default_rng(12)
    a = g.standard_normal((37, 300))
    b = g.standard_normal((53, 300))
    y = oracle_mod.gemm_fprop(a, b)
    ref = a @ b.T
    bound = 300 * 2.0 ** -52 * (np.abs(a) @ np.abs(b).T)
    assert np.all(np.abs(y - ref) <= 2 * bound)
    dx = oracle_mod.gemm_dgrad(a @ b.T, b)          # [37,53] x [53,300]
    assert np.allclose(dx, (a @ b.T) @ b, rtol=1e-12, atol=1e-9)
    dw = oracle_mod.gemm_wgrad(a.T.copy(), a.T.copy())   # [300,37] x [300,37]^T
    assert np.allclose(dw, a.T @ a, rtol=1e-12, atol=1e-9)


def test_gemm_row_selection(oracle_mod):
    g = np.random.default_rng(13)
    a = g.standard_normal((20, 128))
    b = g.standard_normal((16, 128))
    full = oracle_mod.gemm_fprop(a, b)
    part = oracle_mod.gemm_fprop(a, b, rows=[19, 3, 7])
    assert np.array_equal(part, full[[19, 3, 7]])


def test_gemm_identity_weight_is_exact(oracle_mod):
    """W = I quantizes to code 0x78 (256) with scale 2^-8, so Y equals the
    dequantized X exactly, and rounds to BF16 without error (an E4M3 value
    times a power of two has at most 4 significant bits)."""
    x = _rand_bf16((64, 256), 14)
    w = torch.eye(256, dtype=torch.bfloat16)
    qw, sw = oracle_mod.quant_weight(w)
    assert np.all(np.diag(qw) == 0x78) and np.all(np.diag(sw) == 127 - 8)
    qx, sx = oracle_mod.quant_rowwise(x)
    xd = oracle_mod.dequant_groups(qx, sx)
    y = oracle_mod.linear_fprop(x, w)
    assert np.array_equal(y, xd)
    assert np.array_equal(oracle_mod.bf16_to_double(oracle_mod.to_bf16_bits(y)), y)


def test_gemm_all_ones_closed_form(oracle_mod):
    """X = W = 1: scales 2^-8 each, codes 256, Y = K exactly."""
    x = torch.ones(8, 384, dtype=torch.bfloat16)
    w = torch.ones(128, 384, dtype=torch.bfloat16)
    y = oracle_mod.linear_fprop(x, w)
    assert np.all(y == 384.0)


def test_dgrad_and_wgrad_index_order(oracle_mod):
    """dgrad(dY, W) = fprop(dY, W^T) and wgrad(dY^T, X^T) = fprop(dY^T, X^T)
    exactly (same summation order); a transposed operand would break it."""
    g = np.random.default_rng(15)
    dy = g.standard_normal((9, 256))
    w = g.standard_normal((256, 384))
    assert np.array_equal(oracle_mod.gemm_dgrad(dy, w), oracle_mod.gemm_fprop(dy, w.T.copy()))
    dyt = g.standard_normal((5, 130))
    xt = g.standard_normal((7, 130))
    assert np.array_equal(oracle_mod.gemm_wgrad(dyt, xt), oracle_mod.gemm_fprop(dyt, xt))


# ---------------------------------------------------------------- BF16 rounding

def test_bf16_rounding_matches_torch_on_float32_values(oracle_mod):
    """For values exact in binary32, torch's float32->bfloat16 cast is a single
    RNE rounding; the oracle's direct FP64->BF16 rounding must agree."""
    g = torch.Generator().manual_seed(16)
    bits = torch.randint(0, 2 ** 31 - 1, (100000,), generator=g, dtype=torch.int64)
    bits[::4] = (bits[::4] & ~0xFFFF) | 0x8000          # exact ties
    f = bits.to(torch.int32).view(torch.float32)
    f = f[torch.isfinite(f)]
    ref = f.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle_mod.to_bf16_bits(f.double().numpy())
    assert np.array_equal(got, ref)
