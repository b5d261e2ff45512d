"""Several host threads calling the library at once, each on its own stream.

The header allows it: the per-device setup (device checks, kernel attributes,
launch limits) is done once behind a mutex or atomics, and launch parameters
are per call.  The check runs in a fresh process, so that the threads' first
calls race on that setup: four threads start together on four streams, each
runs a whole linear layer (forward, backward into BF16 and into FP32 main
grads) three times on its own shape -- one of them long enough for the
quantizer's ticket schedule, each with its own tile counter -- and every
result must equal, bit for bit, the same layer run afterwards on one thread
and the default stream.
"""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

SCRIPT = r"""
import sys
import threading
import numpy as np
import torch
import fp8_block_scaled_13_b200 as fp8
sys.path.insert(0, "tests")
from helpers import gpu_colwise, gpu_rowwise

shapes = [(300, 384, 256), (4096, 1024, 768), (40000, 1024, 256), (129, 256, 128)]
inputs = []
for i, (m, k, n) in enumerate(shapes):
    g = torch.Generator(device="cuda").manual_seed(100 + i)
    x = (torch.randn(m, k, device="cuda", generator=g) * 2).to(torch.bfloat16)
    w = (torch.randn(n, k, device="cuda", generator=g) * 0.05).to(torch.bfloat16)
    dy = (torch.randn(m, n, device="cuda", generator=g) * 0.1).to(torch.bfloat16)
    inputs.append((x, w, dy))
torch.cuda.synchronize()


def layer(x, w, dy, reps):
    main = torch.zeros(w.shape, dtype=torch.float32, device="cuda")
    for _ in range(reps):
        y, xq, wq = fp8.linear_forward(x, w)
        dx, dw = fp8.linear_backward(dy, xq, wq)
        fp8.linear_backward(dy, xq, wq, main_grad=main)
    torch.cuda.current_stream().synchronize()
    outs = [t.view(torch.int16) if t.dtype == torch.bfloat16 else t
            for t in (y, dx, dw, main, wq.q, wq.s, wq.qt)]
    outs = [t.cpu().numpy() for t in outs]
    # the quantized X, unblocked: only the scale bytes the layout defines
    return outs + list(gpu_rowwise(xq)) + list(gpu_colwise(xq))


results = [None] * len(shapes)
errors = []
start = threading.Barrier(len(shapes))


def worker(i):
    try:
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            start.wait()
            results[i] = layer(*inputs[i], reps=3)
    except BaseException as e:  # reported by the main thread
        errors.append("thread %d: %r" % (i, e))


threads = [threading.Thread(target=worker, args=(i,)) for i in range(len(shapes))]
for t in threads:
    t.start()
for t in threads:
    t.join()
assert not errors, errors
torch.cuda.synchronize()
assert fp8.device_status() == 0

for i in range(len(shapes)):
    want = layer(*inputs[i], reps=3)
    assert len(results[i]) == len(want) == 12
    for j, (a, b) in enumerate(zip(results[i], want)):
        assert a.shape == b.shape and np.array_equal(a, b), \
            "shape %s, output %d differs from the single-thread run" % (shapes[i], j)
print("threads ok")
"""


def test_concurrent_threads_match_one_thread():
    from fp8_block_scaled_13_b200 import build
    build.build()
    env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    assert r.stdout.strip().endswith("threads ok")
