"""Data-parallel weight-gradient exchange (fp8_block_scaled_13_b200.dp) on
two gloo ranks on the CPU.

Each rank takes its own slice of the tokens, computes the partial weight
gradients of two linear layers with the CPU oracle (standing in for the GPU
GEMM, which needs a B200), writes them into the flat FP32 MainGrads buffer,
and the ranks exchange them.  Checks:
  * the summed gradients equal the full-batch gradient: with 128-aligned
    token slices every rank quantizes exactly the full batch's 128-token
    groups (the pages' DP: each rank's micro-batches, gradients combined by
    an all-reduce), and the FP64 partial sums add up to the full sum;
  * the collective itself: the all-reduced buffer is bit-exactly
    fl32(fl32(p0) + fl32(p1)); the average is that / 2; each rank's
    reduce-scatter shard is its slice of the sum; per-layer asynchronous
    exchanges give the same buffer as one whole-buffer exchange;
  * a negative control: slices that are not 128-aligned regroup the tokens
    (token 150 is an outlier, so the full batch's group [128, 256) has a
    coarse scale that tokens 192..255 do not share in the misaligned split),
    and the identity fails by far more than rounding.
"""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

SHAPES = [(256, 384), (128, 256)]   # (n, k) of two layers
M = 512                             # tokens in the full batch


def _inputs():
    g = torch.Generator().manual_seed(1234)
    layers = []
    for (n, k) in SHAPES:
        x = torch.randn(M, k, generator=g)
        x[150] *= 1000.0  # an outlier token: its 128-token group gets a coarse scale
        x = x.to(torch.bfloat16)
        dy = (torch.randn(M, n, generator=g) * 1e-3).to(torch.bfloat16)
        layers.append((x, dy))
    return layers


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, outdir, split):
    import datetime
    import torch.distributed as dist
    import oracle
    from fp8_block_scaled_13_b200.dp import MainGrads

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        layers = _inputs()
        bounds = [0, split, M]
        lo, hi = bounds[rank], bounds[rank + 1]
        grads = MainGrads(SHAPES)
        partial = []
        for i, (x, dy) in enumerate(layers):
            p = oracle.linear_wgrad(dy[lo:hi].contiguous(), x[lo:hi].contiguous())
            partial.append(p)
            grads[i].copy_(torch.from_numpy(p.astype(np.float32)))
        # all partials, for the exact expectations (two-rank sum is order-free)
        gathered = [None] * world
        dist.all_gather_object(gathered, [p for p in partial])
        before = grads.flat.clone()
        grads.all_reduce_(average=False)
        summed = grads.flat.clone()
        result = {"summed": [grads[i].numpy().copy() for i in range(len(SHAPES))],
                  "partials": gathered}
        # average
        grads.flat.copy_(before)
        grads.all_reduce_(average=True)
        result["avg_ok"] = bool(torch.equal(grads.flat, summed / 2))
        # reduce-scatter shard
        grads.flat.copy_(before)
        shard = grads.reduce_scatter(average=False)
        a, b = grads.shard_range(rank)
        result["rs_ok"] = bool(torch.equal(shard, summed[a:b]))
        # per-layer asynchronous exchange
        grads.flat.copy_(before)
        for i in range(len(SHAPES)):
            grads.all_reduce_layer_async(i, average=False)
        grads.wait()
        result["async_ok"] = bool(torch.equal(grads.flat, summed))
        result["full"] = [oracle.linear_wgrad(dy, x) for (x, dy) in layers] if rank == 0 else None
        torch.save(result, os.path.join(outdir, "rank%d.pt" % rank))
    finally:
        dist.destroy_process_group()


def _run(split):
    with tempfile.TemporaryDirectory() as d:
        ctx = mp.get_context("spawn")
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, d, split)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
        for p in procs:
            if p.is_alive():
                p.kill()
                pytest.fail("a gloo rank did not finish")
            assert p.exitcode == 0, "rank exited with %s" % p.exitcode
        return [torch.load(os.path.join(d, "rank%d.pt" % r), weights_only=False) for r in range(2)]


@pytest.fixture(scope="module")
def aligned(oracle_mod):
    return _run(split=256)   # 256 tokens per rank: 128-aligned slices


def test_dp_sum_equals_full_batch_gradient(aligned):
    r0, r1 = aligned
    for i in range(len(SHAPES)):
        p0, p1 = r0["partials"][0][i], r0["partials"][1][i]
        full = r0["full"][i]
        # the FP64 partial sums add up to the full-batch sum (same 128-token groups)
        assert np.max(np.abs((p0 + p1) - full)) <= 1e-12 * np.max(np.abs(full))
        # the exchanged buffer is the FP32 sum of the FP32 partials, on both ranks
        want = (p0.astype(np.float32) + p1.astype(np.float32)).astype(np.float32)
        assert np.array_equal(r0["summed"][i], want)
        assert np.array_equal(r1["summed"][i], want)


def test_dp_average_reduce_scatter_and_async(aligned):
    for r in aligned:
        assert r["avg_ok"] and r["rs_ok"] and r["async_ok"]


def test_dp_misaligned_slices_change_the_quantization(oracle_mod):
    r0, _ = _run(split=192)   # rank 0 gets tokens 0..191: groups [0,128) [128,192)
    p0, p1 = r0["partials"][0][0], r0["partials"][1][0]
    full = r0["full"][0]
    assert np.max(np.abs((p0 + p1) - full)) > 1e-6 * np.max(np.abs(full))


def test_main_grads_layout_single_process():
    from fp8_block_scaled_13_b200.dp import MainGrads
    g = MainGrads([(3, 5), (128, 256), (7, 1)])
    assert len(g) == 3
    for v, (n, k) in zip(g.views, [(3, 5), (128, 256), (7, 1)]):
        assert tuple(v.shape) == (n, k)
        assert v.storage_offset() % 16 == 0
        assert float(v.abs().sum()) == 0.0
    assert g.flat.numel() % 16 == 0
    assert g.shard_range(0) == (0, g.flat.numel())
    g[1].fill_(2.0)
    assert float(g.flat.sum()) == 2.0 * 128 * 256
    assert torch.equal(g.reduce_scatter(), g.flat)
