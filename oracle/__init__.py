"""CPU oracle for the block-scaled FP8 linear layer -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product library never calls it and never falls back to it.

The arithmetic lives in ``puro_oracle.c`` (plain C, FP64, no CUDA); this module
only compiles it (``gcc``) and marshals numpy arrays through ctypes.  BF16
tensors are passed as their uint16 bit patterns.

Sources restated (the Puro-2B report, five web summaries):
  * paper.rainbus.top summary, background "FP8 块级混合精度训练" and
    "方法步骤详情" step (3): E4M3, 1x128 activation groups along the reduction
    dimension, 128x128 weight blocks, one online power-of-two scale per block,
    fprop/dgrad/wgrad in E4M3.
  * ta-paperlens explainer §3.2: activations and gradients grouped by 128
    along the reduction direction, weights by 128x128 blocks.
  * paperlayer.ai summary, Appendix C "FP8 implementation pipeline": the
    forward, data-gradient and weight-gradient GEMMs use blockwise E4M3.

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against closed forms, brute force, exact integer arithmetic and library
routines (torch's float8_e4m3fn cast, numpy matmul on exact inputs).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "puro_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpuro_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile puro_oracle.c into libpuro_oracle.so (gcc, OpenMP, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I = ctypes.c_int64
    lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_double.restype = ctypes.c_double
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    lib.oracle_scale_exponent.argtypes = [ctypes.c_double]
    lib.oracle_scale_exponent.restype = ctypes.c_int
    lib.oracle_double_to_bf16.argtypes = [ctypes.c_double]
    lib.oracle_double_to_bf16.restype = ctypes.c_uint16
    for name in ("oracle_quant_rowwise", "oracle_quant_colwise", "oracle_quant_weight"):
        getattr(lib, name).argtypes = [P, I, I, I, P, P]
        getattr(lib, name).restype = None
    for name in ("oracle_dequant_groups", "oracle_dequant_blocks"):
        getattr(lib, name).argtypes = [P, I, I, P, P]
        getattr(lib, name).restype = None
    for name in ("oracle_gemm_fprop", "oracle_gemm_dgrad", "oracle_gemm_wgrad"):
        getattr(lib, name).argtypes = [P, P, I, I, I, P, I, P]
        getattr(lib, name).restype = None
    lib.oracle_round_bf16_array.argtypes = [P, I, P]
    lib.oracle_round_bf16_array.restype = None
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x) -> np.ndarray:
    """Accept a uint16 numpy array of BF16 bit patterns or a torch bf16 tensor."""
    if hasattr(x, "dtype") and str(x.dtype) == "torch.bfloat16":
        import torch
        x = x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("expected BF16 bit patterns as uint16, got %s" % x.dtype)
    return x


# ---- scalar format helpers -------------------------------------------------

def e4m3_decode(codes) -> np.ndarray:
    """OCP E4M3 value of every code (NaN for 0x7F/0xFF)."""
    lib = _load()
    codes = np.asarray(codes, dtype=np.uint8)
    table = np.array([lib.oracle_e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return table[codes]


def e4m3_encode(values) -> np.ndarray:
    """Round-to-nearest-even, saturating E4M3 code of every value."""
    lib = _load()
    v = np.asarray(values, dtype=np.float64)
    flat = v.reshape(-1)
    out = np.fromiter((lib.oracle_e4m3_encode(float(t)) for t in flat), dtype=np.uint8,
                      count=flat.size)
    return out.reshape(v.shape)


def scale_exponent(amax: float) -> int:
    """Smallest e in [-127, 127] with amax <= 448 * 2^e (0 for amax == 0)."""
    return int(_load().oracle_scale_exponent(float(amax)))


def bf16_to_double(bits) -> np.ndarray:
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """Round FP64 values to BF16 (ties to even); returns uint16 bit patterns."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.shape, dtype=np.uint16)
    _load().oracle_round_bf16_array(_ptr(v), v.size, _ptr(out))
    return out


# ---- quantizers ------------------------------------------------------------

def quant_rowwise(x):
    """1x128 groups along the columns.  Returns (q [R,C] u8, s [R,C/128] u8)."""
    x = _bf16_bits(x)
    R, C = x.shape
    if C % 128:
        raise ValueError("cols must be a multiple of 128")
    q = np.empty((R, C), np.uint8)
    s = np.empty((R, C // 128), np.uint8)
    _load().oracle_quant_rowwise(_ptr(x), R, C, C, _ptr(q), _ptr(s))
    return q, s


def quant_colwise(x):
    """1x128 groups along the rows, output transposed.
    Returns (qt [C,R] u8, st [C,ceil(R/128)] u8)."""
    x = _bf16_bits(x)
    R, C = x.shape
    G = (R + 127) // 128
    qt = np.empty((C, R), np.uint8)
    st = np.empty((C, G), np.uint8)
    _load().oracle_quant_colwise(_ptr(x), R, C, C, _ptr(qt), _ptr(st))
    return qt, st


def quant_weight(w):
    """128x128 blocks.  Returns (q [N,K] u8, s [N/128,K/128] u8)."""
    w = _bf16_bits(w)
    N, K = w.shape
    if N % 128 or K % 128:
        raise ValueError("weight dims must be multiples of 128")
    q = np.empty((N, K), np.uint8)
    s = np.empty((N // 128, K // 128), np.uint8)
    _load().oracle_quant_weight(_ptr(w), N, K, K, _ptr(q), _ptr(s))
    return q, s


def dequant_groups(q, s) -> np.ndarray:
    """decode(q) * 2^(s-127) with one scale per (row, 128-column group)."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    R, C = q.shape
    if s.shape != (R, (C + 127) // 128):
        raise ValueError("scale shape %s does not match codes %s" % (s.shape, q.shape))
    out = np.empty((R, C), np.float64)
    _load().oracle_dequant_groups(_ptr(q), R, C, _ptr(s), _ptr(out))
    return out


def dequant_blocks(q, s) -> np.ndarray:
    """decode(q) * 2^(s-127) with one scale per 128x128 block."""
    q = np.ascontiguousarray(q, np.uint8)
    s = np.ascontiguousarray(s, np.uint8)
    N, K = q.shape
    if s.shape != (N // 128, K // 128):
        raise ValueError("scale shape %s does not match codes %s" % (s.shape, q.shape))
    out = np.empty((N, K), np.float64)
    _load().oracle_dequant_blocks(_ptr(q), N, K, _ptr(s), _ptr(out))
    return out


# ---- GEMMs -----------------------------------------------------------------

def _rows(rows, total):
    if rows is None:
        rows = np.arange(total, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    if rows.size and (rows.min() < 0 or rows.max() >= total):
        raise IndexError("row selection out of range")
    return rows


def gemm_fprop(xd, wd, rows=None) -> np.ndarray:
    """Y[m,n] = sum_k X[m,k] W[n,k] in FP64 (xd [M,K], wd [N,K] dequantized)."""
    xd = np.ascontiguousarray(xd, np.float64)
    wd = np.ascontiguousarray(wd, np.float64)
    M, K = xd.shape
    N = wd.shape[0]
    assert wd.shape[1] == K
    rows = _rows(rows, M)
    y = np.empty((rows.size, N), np.float64)
    _load().oracle_gemm_fprop(_ptr(xd), _ptr(wd), M, N, K, _ptr(rows), rows.size, _ptr(y))
    return y


def gemm_dgrad(dyd, wd, rows=None) -> np.ndarray:
    """dX[m,k] = sum_n dY[m,n] W[n,k] in FP64 (dyd [M,N], wd [N,K])."""
    dyd = np.ascontiguousarray(dyd, np.float64)
    wd = np.ascontiguousarray(wd, np.float64)
    M, N = dyd.shape
    K = wd.shape[1]
    assert wd.shape[0] == N
    rows = _rows(rows, M)
    dx = np.empty((rows.size, K), np.float64)
    _load().oracle_gemm_dgrad(_ptr(dyd), _ptr(wd), M, N, K, _ptr(rows), rows.size, _ptr(dx))
    return dx


def gemm_wgrad(dytd, xtd, rows=None) -> np.ndarray:
    """dW[n,k] = sum_m dY[m,n] X[m,k] in FP64, from dY^T [N,M] and X^T [K,M]."""
    dytd = np.ascontiguousarray(dytd, np.float64)
    xtd = np.ascontiguousarray(xtd, np.float64)
    N, M = dytd.shape
    K = xtd.shape[0]
    assert xtd.shape[1] == M
    rows = _rows(rows, N)
    dw = np.empty((rows.size, K), np.float64)
    _load().oracle_gemm_wgrad(_ptr(dytd), _ptr(xtd), M, N, K, _ptr(rows), rows.size, _ptr(dw))
    return dw


# ---- the linear layer, end to end ------------------------------------------

def linear_fprop(x, w, rows=None):
    """Quantize X (1x128 along K) and W (128x128), then Y = X W^T in FP64."""
    qx, sx = quant_rowwise(x)
    qw, sw = quant_weight(w)
    return gemm_fprop(dequant_groups(qx, sx), dequant_blocks(qw, sw), rows)


def linear_dgrad(dy, w, rows=None):
    """Quantize dY (1x128 along N) and W (128x128), then dX = dY W in FP64."""
    qdy, sdy = quant_rowwise(dy)
    qw, sw = quant_weight(w)
    return gemm_dgrad(dequant_groups(qdy, sdy), dequant_blocks(qw, sw), rows)


def linear_wgrad(dy, x, rows=None):
    """Quantize dY and X along M (tokens), then dW = dY^T X in FP64."""
    qdyt, sdyt = quant_colwise(dy)
    qxt, sxt = quant_colwise(x)
    return gemm_wgrad(dequant_groups(qdyt, sdyt), dequant_groups(qxt, sxt), rows)
