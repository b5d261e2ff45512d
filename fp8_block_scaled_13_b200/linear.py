"""Torch-facing wrappers of the C ABI: allocate outputs with torch, pass device
pointers and the current stream, raise on a non-zero status.  No arithmetic
happens here; every step runs in libpuro_fp8.so.

Layouts (see include/puro_fp8.h):
  * FP8 codes are torch.uint8 tensors (view them as torch.float8_e4m3fn to
    decode); UE8M0 scales are torch.uint8 bytes, scale = 2^(b - 127).
  * Scales a GEMM reads are 1-D uint8 tensors in the blocked layout
    (512-byte chunks of 128 rows x 4 groups; the index formula is in
    include/puro_fp8.h).
  * Transposed (COLWISE) codes are [cols, ld] with ld = rows rounded up to 16.
"""
from __future__ import annotations

import dataclasses
import functools
from dataclasses import dataclass

import torch

from . import _lib


def _round16(n: int) -> int:
    return (n + 15) // 16 * 16


@functools.lru_cache(maxsize=1024)
def blocked_scale_bytes(rows: int, groups: int) -> int:
    return _lib.puro_fp8_blocked_scale_bytes(rows, groups)


def _blocked(rows: int, groups: int, dev) -> torch.Tensor:
    return torch.empty(max(blocked_scale_bytes(rows, groups), 16), dtype=torch.uint8, device=dev)


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream() -> int:
    """The current CUDA stream of the current device, as a cudaStream_t value."""
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


_FIELD_NAMES: dict = {}


def _tensors(obj):
    """The tensors of a wrapper argument: a tensor, or a dataclass's tensor fields."""
    if isinstance(obj, torch.Tensor):
        return (obj,)
    names = _FIELD_NAMES.get(type(obj))
    if names is None:
        if not dataclasses.is_dataclass(obj) or isinstance(obj, type):
            return ()
        names = _FIELD_NAMES[type(obj)] = tuple(f.name for f in dataclasses.fields(obj))
    return tuple(v for v in (getattr(obj, n) for n in names) if isinstance(v, torch.Tensor))


def _on_operand_device(fn):
    """Run a wrapper on the device its tensors live on.  The library launches
    on the current CUDA device and takes the current stream, so operands on
    another device are made current for the call; operands spread over
    several devices are refused."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        operands = (*args, *kwargs.values()) if kwargs else args
        dev = None
        for a in operands:
            for t in _tensors(a):
                if dev is None:
                    dev = t.device
                elif t.device != dev:
                    devs = {t.device for a in operands for t in _tensors(a)}
                    raise ValueError("%s: operands are on different devices (%s)"
                                     % (fn.__name__, ", ".join(sorted(str(d) for d in devs))))
        if dev is not None and dev.type == "cuda" and dev.index != torch.cuda.current_device():
            with torch.cuda.device(dev):
                return fn(*args, **kwargs)
        return fn(*args, **kwargs)
    return wrapper


def _check(status: int, where: str):
    if status != _lib.PURO_OK:
        raise _lib.PuroError(status, where)


def _need(t, what: str):
    if t is None:
        raise ValueError(what)
    return t


def _check_tensor(t: torch.Tensor, shape, dtypes, name: str, min_cols: bool = False):
    """A caller-supplied buffer: CUDA, one of `dtypes`, row-major 2-D of
    `shape` (with min_cols: at least shape[1] columns)."""
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype not in dtypes:
        raise ValueError("%s must be %s, got %s" % (name, " or ".join(map(str, dtypes)), t.dtype))
    ok_shape = (t.dim() == 2 and t.shape[0] == shape[0] and
                (t.shape[1] >= shape[1] if min_cols else t.shape[1] == shape[1]))
    if not ok_shape or (t.numel() and t.stride(1) != 1):
        raise ValueError("%s must be a row-major %s tensor, got %s" % (name, tuple(shape), tuple(t.shape)))


def _check_bytes(t: torch.Tensor, nbytes: int, name: str):
    if not t.is_cuda or t.dtype != torch.uint8 or not t.is_contiguous() or t.numel() < nbytes:
        raise ValueError("%s must be a contiguous CUDA uint8 tensor of at least %d bytes" % (name, nbytes))


def _require(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("%s must be a row-major 2-D tensor" % name)


def _check_row_operand(qa: "QuantAct", name: str):
    """The row-wise codes [rows, cols] and blocked scales (rows x cols/128
    groups) of a QuantAct, sized for the kernel's tensor maps."""
    q = _need(qa.q, "%s was quantized without the row-wise layout" % name)
    _check_tensor(q, (qa.rows, qa.cols), (torch.uint8,), name + ".q", min_cols=True)
    _check_bytes(_need(qa.s, "%s has no row-wise scales" % name),
                 blocked_scale_bytes(qa.rows, qa.cols // 128), name + ".s")


def _check_col_operand(qa: "QuantAct", name: str):
    """The transposed codes [cols, >= rows rounded to 16] and blocked scales
    (cols x ceil(rows/128) groups) of a QuantAct."""
    qt = _need(qa.qt, "%s was quantized without the column-wise layout" % name)
    _check_tensor(qt, (qa.cols, _round16(qa.rows)), (torch.uint8,), name + ".qt", min_cols=True)
    _check_bytes(_need(qa.st, "%s has no column-wise scales" % name),
                 blocked_scale_bytes(qa.cols, (qa.rows + 127) // 128), name + ".st")


def _check_weight(wq: "QuantWeight", fwd: bool):
    """The weight codes and the blocked scales of the GEMM that reads them:
    q [n, k] with s_fwd (n x k/128 groups) for fprop, qt [k, n] with s_bwd
    (k x n/128 groups) for dgrad."""
    if fwd:
        _check_tensor(wq.q, (wq.n, wq.k), (torch.uint8,), "wq.q", min_cols=True)
        _check_bytes(_need(wq.s_fwd, "the weight was quantized without its blocked fprop scales"),
                     blocked_scale_bytes(wq.n, wq.k // 128), "wq.s_fwd")
    else:
        if wq.qt is None or wq.s_bwd is None:
            raise ValueError("the weight was quantized without its transposed copy "
                             "(quant_weight(transpose=True))")
        _check_tensor(wq.qt, (wq.k, wq.n), (torch.uint8,), "wq.qt", min_cols=True)
        _check_bytes(wq.s_bwd, blocked_scale_bytes(wq.k, wq.n // 128), "wq.s_bwd")


@dataclass
class QuantAct:
    """Result of quant_act.  rows/cols describe the BF16 input."""
    rows: int
    cols: int
    q: torch.Tensor | None = None    # [rows, cols] u8
    s: torch.Tensor | None = None    # blocked: rows x cols/128 groups
    qt: torch.Tensor | None = None   # [cols, ld_qt] u8, transposed codes
    st: torch.Tensor | None = None   # blocked: cols x ceil(rows/128) groups
    # two int32 words, zero before first use, that the quantizer may hand its
    # tiles out from (None: static tile schedule); every call leaves them
    # zero.  Calls that may run at the same time need distinct outputs, and so
    # distinct words.
    work: torch.Tensor | None = None


@dataclass
class QuantWeight:
    n: int
    k: int
    q: torch.Tensor                  # [n, k] u8
    s: torch.Tensor                  # [n/128, k/128] u8, compact
    qt: torch.Tensor | None = None   # [k, n] u8
    s_fwd: torch.Tensor | None = None  # blocked: n rows x k/128 groups (fprop B scales)
    s_bwd: torch.Tensor | None = None  # blocked: k rows x n/128 groups (dgrad B scales)


_LAYOUTS = {"rowwise": _lib.PURO_ROWWISE, "colwise": _lib.PURO_COLWISE, "both": _lib.PURO_BOTH}


@_on_operand_device
def quant_act(x: torch.Tensor, layout: str = "both", out: QuantAct | None = None) -> QuantAct:
    """1x128 quantization of an activation/gradient x [rows, cols] (BF16)."""
    _require(x, torch.bfloat16, "x")
    rows, cols = x.shape
    flag = _LAYOUTS.get(layout)
    if flag is None:
        raise ValueError("layout must be one of %s, got %r" % (", ".join(_LAYOUTS), layout))
    dev = x.device
    if out is None:
        out = QuantAct(rows, cols)
        if flag & _lib.PURO_ROWWISE:
            out.q = torch.empty((rows, cols), dtype=torch.uint8, device=dev)
            out.s = _blocked(rows, cols // 128, dev)
        if flag & _lib.PURO_COLWISE:
            out.qt = torch.empty((cols, _round16(rows)), dtype=torch.uint8, device=dev)
            out.st = _blocked(cols, (rows + 127) // 128, dev)
        out.work = torch.zeros(2, dtype=torch.int32, device=dev)
    else:
        if (out.rows, out.cols) != (rows, cols):
            raise ValueError("out was made for a [%d, %d] input" % (out.rows, out.cols))
        if flag & _lib.PURO_ROWWISE:
            _check_tensor(_need(out.q, "out has no row-wise codes"), (rows, cols), (torch.uint8,), "out.q")
            _check_bytes(_need(out.s, "out has no row-wise scales"), blocked_scale_bytes(rows, cols // 128),
                         "out.s")
        if flag & _lib.PURO_COLWISE:
            _check_tensor(_need(out.qt, "out has no transposed codes"), (cols, _round16(rows)),
                          (torch.uint8,), "out.qt", min_cols=True)
            _check_bytes(_need(out.st, "out has no transposed scales"),
                         blocked_scale_bytes(cols, (rows + 127) // 128), "out.st")
        if out.work is not None and (not out.work.is_cuda or out.work.dtype != torch.int32
                                     or not out.work.is_contiguous() or out.work.numel() < 2):
            raise ValueError("out.work must be a contiguous CUDA int32 tensor of at least 2 elements")
    ptr = lambda t: t.data_ptr() if t is not None else None
    st = _lib.puro_fp8_quant_act(
        x.data_ptr(), rows, cols, x.stride(0), flag,
        ptr(out.q), out.q.stride(0) if out.q is not None else 0, ptr(out.s),
        ptr(out.qt), out.qt.stride(0) if out.qt is not None else 0, ptr(out.st),
        ptr(out.work), _stream())
    _check(st, "puro_fp8_quant_act")
    return out


@_on_operand_device
def quant_weight(w: torch.Tensor, transpose: bool = True, out: QuantWeight | None = None) -> QuantWeight:
    """128x128 block quantization of a weight w [n, k] (BF16)."""
    _require(w, torch.bfloat16, "w")
    n, k = w.shape
    dev = w.device
    if out is None:
        out = QuantWeight(
            n, k,
            torch.empty((n, k), dtype=torch.uint8, device=dev),
            torch.empty((n // 128, k // 128), dtype=torch.uint8, device=dev),
            torch.empty((k, n), dtype=torch.uint8, device=dev) if transpose else None,
            _blocked(n, k // 128, dev),
            _blocked(k, n // 128, dev) if transpose else None)
    else:
        if (out.n, out.k) != (n, k):
            raise ValueError("out was made for a [%d, %d] weight" % (out.n, out.k))
        _check_tensor(out.q, (n, k), (torch.uint8,), "out.q")
        _check_bytes(out.s, (n // 128) * (k // 128), "out.s")
        if out.s_fwd is not None:
            _check_bytes(out.s_fwd, blocked_scale_bytes(n, k // 128), "out.s_fwd")
        if out.qt is not None:
            _check_tensor(out.qt, (k, n), (torch.uint8,), "out.qt", min_cols=True)
            if out.s_bwd is not None:
                _check_bytes(out.s_bwd, blocked_scale_bytes(k, n // 128), "out.s_bwd")
    ptr = lambda t: t.data_ptr() if t is not None else None
    st = _lib.puro_fp8_quant_weight(
        w.data_ptr(), n, k, w.stride(0), out.q.data_ptr(), out.q.stride(0), out.s.data_ptr(),
        ptr(out.qt), out.qt.stride(0) if out.qt is not None else 0,
        ptr(out.s_fwd), ptr(out.s_bwd), _stream())
    _check(st, "puro_fp8_quant_weight")
    return out


@_on_operand_device
def gemm_fprop(xq: QuantAct, wq: QuantWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W^T [m, n] BF16 from the ROWWISE quantization of X and the weight's."""
    m, k, n = xq.rows, xq.cols, wq.n
    if wq.k != k:
        raise ValueError("inner dimensions differ: %d vs %d" % (k, wq.k))
    _check_row_operand(xq, "xq")
    _check_weight(wq, fwd=True)
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=xq.q.device)
    _check_tensor(out, (m, n), (torch.bfloat16,), "out", min_cols=False)
    st = _lib.puro_fp8_gemm_fprop(
        xq.q.data_ptr(), xq.q.stride(0), xq.s.data_ptr(),
        wq.q.data_ptr(), wq.q.stride(0), wq.s_fwd.data_ptr(),
        out.data_ptr(), out.stride(0), m, n, k, _stream())
    _check(st, "puro_fp8_gemm_fprop")
    return out


@_on_operand_device
def gemm_dgrad(dyq: QuantAct, wq: QuantWeight, out: torch.Tensor | None = None) -> torch.Tensor:
    """dX = dY W [m, k] BF16 from the ROWWISE quantization of dY and W's transposed codes."""
    m, n, k = dyq.rows, dyq.cols, wq.k
    if wq.n != n:
        raise ValueError("dY has %d columns, W has %d rows" % (n, wq.n))
    _check_weight(wq, fwd=False)
    _check_row_operand(dyq, "dyq")
    if out is None:
        out = torch.empty((m, k), dtype=torch.bfloat16, device=dyq.q.device)
    _check_tensor(out, (m, k), (torch.bfloat16,), "out")
    st = _lib.puro_fp8_gemm_dgrad(
        dyq.q.data_ptr(), dyq.q.stride(0), dyq.s.data_ptr(),
        wq.qt.data_ptr(), wq.qt.stride(0), wq.s_bwd.data_ptr(),
        out.data_ptr(), out.stride(0), m, n, k, _stream())
    _check(st, "puro_fp8_gemm_dgrad")
    return out


@_on_operand_device
def gemm_wgrad(dyq: QuantAct, xq: QuantAct, out: torch.Tensor | None = None,
               accumulate: bool = False) -> torch.Tensor:
    """dW = dY^T X [n, k] from the COLWISE quantizations of dY and X.

    `out` BF16 (default) or FP32.  With an FP32 `out` and accumulate=True the
    product is added to it (dW += dY^T X, an FP32 gradient buffer); only the
    FP32 output accumulates."""
    m, n, k = dyq.rows, dyq.cols, xq.cols
    if xq.rows != m:
        raise ValueError("dY and X have different token counts")
    if out is None and accumulate:
        raise ValueError("accumulate=True needs the FP32 buffer to add into")
    _check_col_operand(dyq, "dyq")
    _check_col_operand(xq, "xq")
    if out is None:
        out = torch.empty((n, k), dtype=torch.bfloat16, device=dyq.qt.device)
    _check_tensor(out, (n, k), (torch.bfloat16, torch.float32), "out")
    if out.dtype == torch.float32:
        st = _lib.puro_fp8_gemm_wgrad_f32(
            dyq.qt.data_ptr(), dyq.qt.stride(0), dyq.st.data_ptr(),
            xq.qt.data_ptr(), xq.qt.stride(0), xq.st.data_ptr(),
            out.data_ptr(), out.stride(0), m, n, k, 1 if accumulate else 0, _stream())
        _check(st, "puro_fp8_gemm_wgrad_f32")
        return out
    if out.dtype != torch.bfloat16 or accumulate:
        raise ValueError("out must be BF16, or FP32 (required for accumulate=True)")
    st = _lib.puro_fp8_gemm_wgrad(
        dyq.qt.data_ptr(), dyq.qt.stride(0), dyq.st.data_ptr(),
        xq.qt.data_ptr(), xq.qt.stride(0), xq.st.data_ptr(),
        out.data_ptr(), out.stride(0), m, n, k, _stream())
    _check(st, "puro_fp8_gemm_wgrad")
    return out


@_on_operand_device
def gemm_dgrad_wgrad(dyq: QuantAct, wq: QuantWeight, xq: QuantAct, dx: torch.Tensor | None = None,
                     dw: torch.Tensor | None = None, accumulate: bool = False):
    """dX = dY W and dW = dY^T X in one launch (tiles of both spread over the
    GPU together); results identical to gemm_dgrad and gemm_wgrad.  `dw` BF16
    (default) or FP32; accumulate=True adds into an FP32 `dw`.  Returns (dx, dw)."""
    m, n, k = dyq.rows, dyq.cols, wq.k
    if wq.n != n or xq.rows != m or xq.cols != k:
        raise ValueError("shapes of dY, W and X do not agree")
    if dw is None and accumulate:
        raise ValueError("accumulate=True needs the FP32 buffer to add into")
    _check_weight(wq, fwd=False)
    _check_row_operand(dyq, "dyq")
    _check_col_operand(dyq, "dyq")
    _check_col_operand(xq, "xq")
    dev = dyq.q.device
    if dx is None:
        dx = torch.empty((m, k), dtype=torch.bfloat16, device=dev)
    if dw is None:
        if accumulate:
            raise ValueError("accumulate=True needs the FP32 buffer to add into")
        dw = torch.empty((n, k), dtype=torch.bfloat16, device=dev)
    _check_tensor(dx, (m, k), (torch.bfloat16,), "dx")
    _check_tensor(dw, (n, k), (torch.bfloat16, torch.float32), "dw")
    if dw.dtype == torch.float32:
        kind = _lib.PURO_DW_F32_ACCUMULATE if accumulate else _lib.PURO_DW_F32
    elif dw.dtype == torch.bfloat16 and not accumulate:
        kind = _lib.PURO_DW_BF16
    else:
        raise ValueError("dw must be BF16, or FP32 (required for accumulate=True)")
    st = _lib.puro_fp8_gemm_dgrad_wgrad(
        dyq.q.data_ptr(), dyq.q.stride(0), dyq.s.data_ptr(),
        wq.qt.data_ptr(), wq.qt.stride(0), wq.s_bwd.data_ptr(),
        dx.data_ptr(), dx.stride(0),
        dyq.qt.data_ptr(), dyq.qt.stride(0), dyq.st.data_ptr(),
        xq.qt.data_ptr(), xq.qt.stride(0), xq.st.data_ptr(),
        dw.data_ptr(), dw.stride(0), m, n, k, kind, _stream())
    _check(st, "puro_fp8_gemm_dgrad_wgrad")
    return dx, dw


def device_status() -> int:
    """Synchronize the current stream and return/clear the device error word."""
    return _lib.puro_fp8_device_status(_stream())


def linear_forward(x: torch.Tensor, w: torch.Tensor | None = None, wq: QuantWeight | None = None):
    """Quantize X (and W, unless its quantization `wq` is passed in), then
    Y = X W^T.  Returns (y, xq, wq).

    Passing the previous call's `wq` skips re-quantizing a weight that has not
    changed, e.g. across the micro-batches of one gradient-accumulation step
    (the codes would be identical)."""
    if wq is None:
        if w is None:
            raise ValueError("pass the weight or its quantization")
        wq = quant_weight(w, transpose=True)
    xq = quant_act(x, "both")
    return gemm_fprop(xq, wq), xq, wq


def linear_backward(dy: torch.Tensor, xq: QuantAct, wq: QuantWeight,
                    main_grad: torch.Tensor | None = None):
    """Quantize dY both ways, then dX = dY W and dW = dY^T X.  Returns (dx, dw).

    With `main_grad` (FP32 [n, k]) the weight gradient is added into it
    (gradient accumulation across micro-batches) and returned as dw."""
    dyq = quant_act(dy, "both")
    if main_grad is not None:
        return gemm_dgrad_wgrad(dyq, wq, xq, dw=main_grad, accumulate=True)
    return gemm_dgrad_wgrad(dyq, wq, xq)
