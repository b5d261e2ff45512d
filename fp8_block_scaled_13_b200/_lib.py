"""ctypes binding of libpuro_fp8.so: the C ABI of include/puro_fp8.h, same names.

Argument marshalling only.  Every pointer is an integer device address and
every stream an integer cudaStream_t.  There is no fallback: if the library is
missing or the device is not a B200 the calls fail loudly.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpuro_fp8.so")

PURO_OK = 0
PURO_ERR_NULL = -1
PURO_ERR_ALIGN = -2
PURO_ERR_SHAPE = -3
PURO_ERR_LAYOUT = -4
PURO_ERR_CUDA = -5
PURO_ERR_UNSUPPORTED_DEVICE = -6
PURO_ERR_DEVICE_TIMEOUT = -7

PURO_ROWWISE = 1
PURO_COLWISE = 2
PURO_BOTH = 3
PURO_DW_BF16 = 0
PURO_DW_F32 = 1
PURO_DW_F32_ACCUMULATE = 2

EXPORTS = (
    "puro_fp8_blocked_scale_bytes",
    "puro_fp8_quant_act",
    "puro_fp8_quant_act_static_scratch",
    "puro_fp8_quant_weight",
    "puro_fp8_gemm_fprop",
    "puro_fp8_gemm_dgrad",
    "puro_fp8_gemm_wgrad",
    "puro_fp8_gemm_wgrad_f32",
    "puro_fp8_gemm_dgrad_wgrad",
    "puro_fp8_device_status",
    "puro_fp8_status_string",
    "puro_fp8_test_bounded_wait",
    "puro_fp8_test_schedule",
)

_lib = None


class PuroError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = status
        super().__init__("%s%s" % (where + ": " if where else "", status_string(status)))


def load() -> ctypes.CDLL:
    """Load the CUDA library (raises if it was not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            "libpuro_fp8.so is missing (%s); build it with "
            "`python -c 'import __graft_entry__ as g; g.build()'`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P, I, INT = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.puro_fp8_blocked_scale_bytes.argtypes = [I, I]
    lib.puro_fp8_blocked_scale_bytes.restype = I
    lib.puro_fp8_quant_act.argtypes = [P, I, I, I, INT, P, I, P, P, I, P, P, P]
    lib.puro_fp8_quant_act_static_scratch.argtypes = [P, I, I, I, INT, P, I, P, P, I, P, P]
    lib.puro_fp8_quant_weight.argtypes = [P, I, I, I, P, I, P, P, I, P, P, P]
    lib.puro_fp8_gemm_fprop.argtypes = [P, I, P, P, I, P, P, I, I, I, I, P]
    lib.puro_fp8_gemm_dgrad.argtypes = [P, I, P, P, I, P, P, I, I, I, I, P]
    lib.puro_fp8_gemm_wgrad.argtypes = [P, I, P, P, I, P, P, I, I, I, I, P]
    lib.puro_fp8_gemm_wgrad_f32.argtypes = [P, I, P, P, I, P, P, I, I, I, I, INT, P]
    lib.puro_fp8_gemm_dgrad_wgrad.argtypes = [P, I, P, P, I, P, P, I, P, I, P, P, I, P, P, I,
                                              I, I, I, INT, P]
    lib.puro_fp8_device_status.argtypes = [P]
    lib.puro_fp8_status_string.argtypes = [INT]
    lib.puro_fp8_status_string.restype = ctypes.c_char_p
    lib.puro_fp8_test_bounded_wait.argtypes = [I, P]
    I32 = ctypes.c_int32
    lib.puro_fp8_test_schedule.argtypes = [I32, I32, I32, I32, I32, P, P]
    for name in EXPORTS:
        if name not in ("puro_fp8_status_string", "puro_fp8_blocked_scale_bytes"):
            getattr(lib, name).restype = INT
    _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().puro_fp8_status_string(int(status)).decode()


def puro_fp8_blocked_scale_bytes(rows, groups) -> int:
    return load().puro_fp8_blocked_scale_bytes(rows, groups)


def puro_fp8_quant_act(x, rows, cols, ld_x, layout, q, ld_q, s, qt, ld_qt, st, tile_counter,
                       stream) -> int:
    return load().puro_fp8_quant_act(x, rows, cols, ld_x, layout, q, ld_q, s, qt, ld_qt, st,
                                     tile_counter, stream)


def puro_fp8_quant_weight(w, n, k, ld_w, q, ld_q, s, qt, ld_qt, s_fwd, s_bwd, stream) -> int:
    return load().puro_fp8_quant_weight(w, n, k, ld_w, q, ld_q, s, qt, ld_qt, s_fwd, s_bwd, stream)


def puro_fp8_gemm_fprop(qx, ld_qx, sx, qw, ld_qw, sw_fwd, y, ld_y, m, n, k, stream) -> int:
    return load().puro_fp8_gemm_fprop(qx, ld_qx, sx, qw, ld_qw, sw_fwd, y, ld_y, m, n, k, stream)


def puro_fp8_gemm_dgrad(qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx, m, n, k, stream) -> int:
    return load().puro_fp8_gemm_dgrad(qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx, m, n, k,
                                      stream)


def puro_fp8_gemm_wgrad(qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k, stream) -> int:
    return load().puro_fp8_gemm_wgrad(qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k,
                                      stream)


def puro_fp8_gemm_wgrad_f32(qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k, accumulate,
                            stream) -> int:
    return load().puro_fp8_gemm_wgrad_f32(qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k,
                                          accumulate, stream)


def puro_fp8_gemm_dgrad_wgrad(qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx, qdyt, ld_qdyt, sdyt,
                              qxt, ld_qxt, sxt, dw, ld_dw, m, n, k, dw_kind, stream) -> int:
    return load().puro_fp8_gemm_dgrad_wgrad(qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx, qdyt,
                                            ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k,
                                            dw_kind, stream)


def puro_fp8_device_status(stream) -> int:
    return load().puro_fp8_device_status(stream)


def puro_fp8_status_string(status) -> str:
    return status_string(status)


def puro_fp8_test_bounded_wait(limit_ns, stream) -> int:
    return load().puro_fp8_test_bounded_wait(limit_ns, stream)


def puro_fp8_test_schedule(units0, kblocks0, units1, kblocks1, clusters, offsets, units) -> int:
    return load().puro_fp8_test_schedule(units0, kblocks0, units1, kblocks1, clusters, offsets,
                                         units)
