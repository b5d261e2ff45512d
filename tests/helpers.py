"""Shared helpers of the GPU parity tests (comparison and tolerance logic)."""
from __future__ import annotations

import numpy as np
import torch


def np_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def blocked_index(rows: int, groups: int) -> np.ndarray:
    """[rows, groups] matrix of byte offsets into a blocked scale array
    (the index formula of include/puro_fp8.h)."""
    r = np.arange(rows, dtype=np.int64)[:, None]
    g = np.arange(groups, dtype=np.int64)[None, :]
    g4 = (groups + 3) // 4
    return ((r // 128) * g4 + g // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + g % 4


def unblock(s, rows: int, groups: int) -> np.ndarray:
    """Blocked scale array -> [rows, groups] matrix."""
    s = np_u8(s) if hasattr(s, "cpu") else np.asarray(s)
    return s.reshape(-1)[blocked_index(rows, groups)]


def gpu_rowwise(xq, rows=None):
    """(q [R,C], s [R,G]) in the oracle's orientation from a QuantAct."""
    R, C = xq.rows, xq.cols
    q = np_u8(xq.q)
    s = unblock(xq.s, R, C // 128)
    if rows is not None:
        q, s = q[rows], s[rows]
    return q, s


def gpu_colwise(xq):
    """(qt [C,R], st [C,G]) in the oracle's orientation, plus the zero padding."""
    R, C = xq.rows, xq.cols
    qt_full = np_u8(xq.qt)
    st = unblock(xq.st, C, (R + 127) // 128)
    pad = qt_full[:, R:(R + 15) // 16 * 16]
    return qt_full[:, :R], st, pad


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return np.exp2(np.floor(np.log2(a)) - 7)


def gemm_errors(got: torch.Tensor, ref64: np.ndarray, oracle):
    """Relative Frobenius error against the oracle's BF16-rounded result, and
    the worst excess of |got - ref| over 4e-3*rms(ref) + 1 BF16 ulp(ref)."""
    g = got.detach().float().cpu().numpy().astype(np.float64)
    ref_bf16 = oracle.bf16_to_double(oracle.to_bf16_bits(ref64))
    den = np.linalg.norm(ref_bf16)
    rel = np.linalg.norm(g - ref_bf16) / den if den > 0 else np.linalg.norm(g)
    rms = np.sqrt(np.mean(ref64 ** 2)) if ref64.size else 0.0
    excess = np.abs(g - ref64) - (4e-3 * rms + bf16_ulp(ref64))
    return float(rel), float(excess.max()) if excess.size else -1.0


def assert_gemm_close(got, ref64, oracle, what=""):
    rel, excess = gemm_errors(got, ref64, oracle)
    assert rel <= 1e-3, "%s: relative Frobenius error %.3g > 1e-3" % (what, rel)
    assert excess <= 0.0, "%s: an element exceeds 4e-3*rms + 1 ulp by %.3g" % (what, excess)
    return rel


def assert_f32_close(got, ref64: np.ndarray, init=None, what=""):
    """FP32-output GEMM check: relative Frobenius error <= 1e-3 of the FP64
    product, and every element within 4e-3 * rms(product) + 1 FP32 ulp of the
    expected value (init + product when the output was accumulated into)."""
    g = got.detach().cpu().numpy().astype(np.float64)
    exp = ref64 if init is None else np.asarray(init, dtype=np.float64) + ref64
    den = np.linalg.norm(ref64)
    rel = np.linalg.norm(g - exp) / den if den > 0 else np.linalg.norm(g - exp)
    assert rel <= 1e-3, "%s: relative Frobenius error %.3g > 1e-3" % (what, rel)
    rms = np.sqrt(np.mean(ref64 ** 2)) if ref64.size else 0.0
    ulp = np.spacing(np.abs(exp).astype(np.float32)).astype(np.float64)
    excess = np.abs(g - exp) - (4e-3 * rms + ulp)
    assert excess.max() <= 0.0, "%s: an element exceeds the tolerance by %.3g" % (what, excess.max())
    return rel
