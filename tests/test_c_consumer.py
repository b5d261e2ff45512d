"""The C ABI from a plain C99 program (tests/c_abi/abi_consumer.c): the header
compiles as strict C99 and as C++17, a C program links the library with no
Python or torch in the process, gets the documented argument errors (CPU), and
runs one linear layer on device buffers it allocates itself, checked against
the oracle (GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "abi_consumer.c")
INCLUDE = os.path.join(ROOT, "include")
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")
STRICT = ["-std=c99", "-O1", "-Wall", "-Wextra", "-Werror", "-pedantic"]


def _product_lib():
    from fp8_block_scaled_13_b200 import build
    return build.build()


def _oracle_lib():
    import oracle
    return oracle.build()


def _compile(out, gpu):
    lib = _product_lib()
    libdirs = [os.path.dirname(lib)]
    cmd = ["gcc", *STRICT, "-I" + INCLUDE, SRC, "-L" + libdirs[0], "-lpuro_fp8"]
    if gpu:
        orc = _oracle_lib()
        libdirs += [os.path.dirname(orc), os.path.join(CUDA, "lib64")]
        # the CUDA headers are not strict C99: include them as system headers
        cmd[1:1] = ["-DABI_CONSUMER_GPU", "-isystem", os.path.join(CUDA, "include")]
        cmd += ["-L" + libdirs[1], "-lpuro_oracle", "-L" + libdirs[2], "-lcudart"]
    cmd += ["-Wl,-rpath," + ":".join(libdirs), "-lm", "-o", out]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_header_compiles_as_c99_and_cxx17(tmp_path):
    for lang, std in (("c", "c99"), ("c++", "c++17")):
        subprocess.run(["gcc" if lang == "c" else "g++", "-std=" + std, "-Wall", "-Wextra",
                        "-Werror", "-pedantic", "-fsyntax-only", "-x", lang,
                        os.path.join(INCLUDE, "puro_fp8.h")], check=True)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
def test_c_program_host_checks(tmp_path):
    exe = _compile(str(tmp_path / "host"), gpu=False)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip().endswith("abi_consumer: host ok")


@pytest.mark.skipif(shutil.which("gcc") is None or
                    not os.path.exists(os.path.join(CUDA, "include", "cuda_runtime_api.h")),
                    reason="gcc or the CUDA runtime headers not available")
def test_c_program_gpu_mode_builds(tmp_path):
    # compiled and linked everywhere; run only on a GPU (below)
    assert os.path.exists(_compile(str(tmp_path / "gpu"), gpu=True))


@pytest.mark.gpu
def test_c_program_runs_the_layer_on_the_gpu(tmp_path):
    exe = _compile(str(tmp_path / "gpu"), gpu=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("abi_consumer: gpu ok")
