"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/puro_fp8.h declares, and rejects bad arguments
before touching CUDA.  Also checks that the product code never imports the
oracle."""
import ast
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "puro_fp8.h")


@pytest.fixture(scope="module")
def lib():
    from fp8_block_scaled_13_b200 import build, _lib
    build.build()
    return _lib


def _declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"PURO_API\s+(?:const\s+)?\w+\*?\s+\*?(puro_fp8_\w+)\s*\(", src)))


def test_header_declares_the_abi():
    names = _declared()
    for must in ("puro_fp8_quant_act", "puro_fp8_quant_weight", "puro_fp8_gemm_fprop",
                 "puro_fp8_gemm_dgrad", "puro_fp8_gemm_wgrad", "puro_fp8_device_status",
                 "puro_fp8_status_string"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r" T (\w+)", out))
    assert set(_declared()) <= exported
    # nothing else leaks out (the static CUDA runtime stays hidden)
    assert {s for s in exported if not s.startswith("puro_fp8_")} <= {"_init", "_fini"}
    assert set(lib.EXPORTS) == set(_declared())


def test_status_strings(lib):
    for code in range(0, -8, -1):
        s = lib.status_string(code)
        assert s.startswith("PURO_")
    assert "unknown" in lib.status_string(-99)


A = 1 << 20  # a 16-byte-aligned fake device address; never dereferenced here


@pytest.mark.parametrize("args,code", [
    # (x, rows, cols, ld_x, layout, q, ld_q, s, qt, ld_qt, st[, tile_counter])
    ((A, 16, 128, 128, 7, A, 128, A, None, 0, None), -4),     # bad layout flag
    ((A, 16, 100, 128, 1, A, 128, A, None, 0, None), -3),     # cols not a multiple of 128
    ((A, -1, 128, 128, 1, A, 128, A, None, 0, None), -3),     # negative rows
    ((None, 16, 128, 128, 1, A, 128, A, None, 0, None), -1),  # null input
    ((A + 2, 16, 128, 128, 1, A, 128, A, None, 0, None), -2), # misaligned input pointer
    ((A, 16, 256, 128, 1, A, 256, A, None, 0, None), -3),     # ld_x < cols
    ((A, 16, 128, 132, 1, A, 128, A, None, 0, None), -2),     # ld_x*2 not a multiple of 16
    ((A, 16, 128, 128, 1, None, 128, A, None, 0, None), -1),  # ROWWISE without q
    ((A, 16, 128, 128, 1, A, 128, None, None, 0, None), -1),  # ROWWISE without s
    ((A, 16, 128, 128, 1, A, 128, A + 8, None, 0, None), -2), # misaligned s
    ((A, 17, 128, 128, 2, None, 0, None, A, 16, A), -3),      # qt leading dim below rows rounded to 16
    ((A, 16, 128, 128, 2, None, 0, None, A, 16, None), -1),   # COLWISE without st
    ((A, 16, 128, 128, 1, A, 128, A, None, 0, None, A + 4), -2),  # tile counter not 8-byte aligned
])
def test_quant_act_argument_errors(lib, args, code):
    args = args + (None,) * (12 - len(args))
    assert lib.puro_fp8_quant_act(*args, None) == code


def test_quant_act_empty_is_noop(lib):
    assert lib.puro_fp8_quant_act(None, 0, 128, 128, 3, None, 0, None, None, 0, None, None, None) == 0
    assert lib.puro_fp8_quant_act(None, 5, 0, 0, 3, None, 0, None, None, 0, None, None, None) == 0


@pytest.mark.parametrize("args,code", [
    # (w, n, k, ld_w, q, ld_q, s, qt, ld_qt, s_fwd, s_bwd)
    ((A, 100, 128, 128, A, 128, A, None, 0, A, None), -3),     # n not multiple of 128
    ((A, 128, 100, 128, A, 128, A, None, 0, A, None), -3),     # k not multiple of 128
    ((A, 128, 128, 128, None, 128, A, None, 0, A, None), -1),  # q null
    ((A, 128, 128, 128, A, 128, None, None, 0, A, None), -1),  # s null
    ((A, 128, 128, 128, A, 128, A, A, 64, A, A), -3),          # ld_qt < n
    ((A, 128, 128, 128, A + 8, 128, A, None, 0, A, None), -2), # misaligned q
    ((A, 128, 128, 128, A, 128, A, None, 0, A + 4, None), -2), # misaligned s_fwd
])
def test_quant_weight_argument_errors(lib, args, code):
    assert lib.puro_fp8_quant_weight(*args, None) == code


@pytest.mark.parametrize("fn,args,code", [
    # fprop/dgrad: (a, lda, sa, b, ldb, sb, d, ldd, m, n, k)
    ("fprop", (A, 256, A, A, 256, A, A, 320, 64, 320, 256), -3),    # n % 128
    ("fprop", (A, 256, A, A, 256, A, A, 256, 64, 256, 200), -3),    # k % 128
    ("fprop", (A, 256, A, A, 256, None, A, 256, 64, 256, 256), -1), # sw_fwd null
    ("fprop", (A, 256, A, A, 256, A + 2, A, 256, 64, 256, 256), -2),# sw_fwd misaligned
    ("fprop", (A, 256, A, A, 256, A, A, 100, 64, 256, 256), -3),    # ld_y < n
    ("fprop", (A, 256, A, A, 256, A, A + 4, 256, 64, 256, 256), -2),
    ("fprop", (A, 128, A, A, 256, A, A, 256, 64, 256, 256), -3),    # ld_qx < k
    ("dgrad", (A, 128, A, A, 256, A, A, 256, 64, 256, 256), -3),    # ld_qdy < n
    ("dgrad", (A, 256, None, A, 256, A, A, 256, 64, 256, 256), -1), # sdy null
    ("wgrad", (A, 48, A, A, 64, A, A, 256, 64, 256, 256), -3),      # ld_qdyt < m
    ("wgrad", (A, 64, A, A, 64, A, A, 256, 64, 200, 256), -3),      # n % 128
    ("wgrad", (A, 64, A, A, 64, None, A, 256, 64, 256, 256), -1),   # sxt null
])
def test_gemm_argument_errors(lib, fn, args, code):
    f = getattr(lib, "puro_fp8_gemm_" + fn)
    assert f(*args, None) == code


@pytest.mark.parametrize("args,code", [
    # (qdyt, ld_qdyt, sdyt, qxt, ld_qxt, sxt, dw, ld_dw, m, n, k, accumulate)
    ((A, 64, A, A, 64, A, A, 256, 64, 256, 256, 2), -4),     # accumulate flag not 0/1
    ((A, 64, A, A, 64, A, A, 258, 64, 256, 256, 0), -2),     # ld_dw * 4 not a multiple of 16
    ((A, 64, A, A, 64, A, A, 128, 64, 256, 256, 1), -3),     # ld_dw < k
    ((A, 64, A, A, 64, A, A, 256, 64, 200, 256, 0), -3),     # n % 128
    ((A, 64, A, A, 64, A, A + 8, 256, 64, 256, 256, 1), -2), # dw misaligned
    ((A, 48, A, A, 64, A, A, 256, 64, 256, 256, 0), -3),     # ld_qdyt < m
    ((A, 64, None, A, 64, A, A, 256, 64, 256, 256, 1), -1),  # sdyt null
])
def test_wgrad_f32_argument_errors(lib, args, code):
    assert lib.puro_fp8_gemm_wgrad_f32(*args, None) == code


def _dw_args(**over):
    # dgrad (qdy, ld_qdy, sdy, qwt, ld_qwt, sw_bwd, dx, ld_dx), wgrad (qdyt, ld_qdyt, sdyt, qxt,
    # ld_qxt, sxt, dw, ld_dw), m, n, k, dw_kind
    a = dict(qdy=A, ld_qdy=256, sdy=A, qwt=A, ld_qwt=256, sw=A, dx=A, ld_dx=256,
             qdyt=A, ld_qdyt=64, sdyt=A, qxt=A, ld_qxt=64, sxt=A, dw=A, ld_dw=256,
             m=64, n=256, k=256, kind=0)
    a.update(over)
    return tuple(a.values())


@pytest.mark.parametrize("over,code", [
    (dict(kind=3), -4),                 # unknown dW kind
    (dict(kind=-1), -4),
    (dict(n=200), -3),                  # n % 128
    (dict(sw=None), -1),                # the dgrad part's checks
    (dict(ld_dx=100), -3),
    (dict(sxt=None), -1),               # the wgrad part's checks
    (dict(ld_dw=258, kind=1), -2),      # FP32 dW row stride not a multiple of 16 bytes
    (dict(ld_qdyt=48), -3),
])
def test_dgrad_wgrad_argument_errors(lib, over, code):
    assert lib.puro_fp8_gemm_dgrad_wgrad(*_dw_args(**over), None) == code


def test_gemm_empty_is_noop(lib):
    assert lib.puro_fp8_gemm_fprop(None, 0, None, None, 0, None, None, 0, 0, 256, 256, None) == 0
    assert lib.puro_fp8_gemm_wgrad(None, 0, None, None, 0, None, None, 0, 64, 0, 256, None) == 0
    assert lib.puro_fp8_gemm_wgrad_f32(None, 0, None, None, 0, None, None, 0, 64, 0, 256, 1,
                                       None) == 0
    # n == 0: both the data and the weight gradient are empty
    assert lib.puro_fp8_gemm_dgrad_wgrad(*_dw_args(n=0, k=0), None) == 0


@pytest.mark.parametrize("rows,groups,want", [
    (0, 4, 0), (4, 0, 0), (1, 1, 512), (128, 4, 512), (129, 4, 1024), (128, 5, 1024),
    (8192, 16, 64 * 4 * 512), (8000, 63, 63 * 16 * 512),
])
def test_blocked_scale_bytes(lib, rows, groups, want):
    assert lib.puro_fp8_blocked_scale_bytes(rows, groups) == want


def _imports(path):
    tree = ast.parse(open(path).read())
    mods = set()
    for node in ast.walk(tree):
        if isinstance(node, ast.Import):
            mods |= {a.name.split(".")[0] for a in node.names}
        elif isinstance(node, ast.ImportFrom) and node.module and node.level == 0:
            mods.add(node.module.split(".")[0])
    return mods


def test_product_never_imports_oracle():
    pkg = os.path.join(ROOT, "fp8_block_scaled_13_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith(".py"):
                assert "oracle" not in _imports(os.path.join(dirpath, f)), f
            if f.endswith((".cu", ".cuh", ".h", ".c", ".cpp")):
                assert "puro_oracle" not in open(os.path.join(dirpath, f)).read(), f


def test_oracle_never_imports_product():
    odir = os.path.join(ROOT, "oracle")
    for f in os.listdir(odir):
        if f.endswith(".py"):
            assert "fp8_block_scaled_13_b200" not in _imports(os.path.join(odir, f))
        if f.endswith(".c"):
            src = open(os.path.join(odir, f)).read()
            includes = re.findall(r'#include\s*[<"]([^>"]+)', src)
            assert not any("puro_fp8" in h or h.startswith("cuda") for h in includes), includes


def test_static_scratch_entry_rejects_before_cuda(lib):
    """The allocation-free quantizer entry point checks its sizes before it
    touches the device: a bad layout, a bad shape, and an input of 2^31 or
    more tiles (the tile counter's limit) come back as errors, and an empty
    input is a no-op."""
    f = lib.load().puro_fp8_quant_act_static_scratch
    args = lambda rows, cols, layout: (A, rows, cols, cols, layout, A, cols, A, A, 16, A, None)
    assert f(*args(16, 128, 7)) == -4
    assert f(*args(16, 100, 3)) == -3
    assert f(*args(-1, 128, 3)) == -3
    assert f(*args(32768, (1 << 31) - 128, 3)) == -3
    assert f(*args(0, 128, 3)) == 0
