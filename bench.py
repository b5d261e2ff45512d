"""Benchmark of the block-scaled FP8 linear layer hot path on B200.

One step = one micro-batch of the attention-projection workload (M = 8192
tokens, hidden 2048; the fused QKV projection 2048->3072 and the output
projection 2048->2048), for each of the two layers:
  quant_act(X, both), fprop, quant_act(dY, both), and one launch computing
  dgrad and wgrad (dW added into FP32 main grads); quant_weight(W) (+
  transposed codes) runs once per gradient-accumulation window of --accum
  steps, since the weights only change at the optimizer step.
value = GEMM FLOPs of the step (2*M*N*K per GEMM, three GEMMs per layer)
divided by the device time of the whole step (quantizers included).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--accum A]
                       [--impl ours|reference]
With N > 1 (torchrun) every rank runs its own batch (data parallel, weak
scaling) and every A steps the ranks all-reduce the FP32 weight gradients.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FP8 block-scaled GEMM TFLOP/s (fprop/dgrad/wgrad) and % of B200 FP8 peak"
WORKLOAD = "attn_proj_m8192_h2048_qkv3072_o2048"
SEED = 1
M_TOKENS = 8192
# dram__bytes_read.sum + dram__bytes_write.sum of one GEMM launch (the QKV
# layer's fprop, 8192 x 3072 x 2048) from an ncu capture of this step; to be
# set to None when the GEMM kernel changes until it is captured again.
GEMM_TRAFFIC_BYTES = 23338496 + 6511104
# The same for one activation quantizer launch (quant_act BOTH of X [8192, 2048]);
# its codes mostly stay in L2 for the GEMM that reads them next, so the DRAM
# traffic is about half the algorithmic bytes.
QUANT_TRAFFIC_BYTES = 33584896 + 833536


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ceiling", action="store_true")
    ap.add_argument("--no-bf16", action="store_true")
    ap.add_argument("--accum", type=int, default=64,
                    help="micro-batch steps per gradient exchange (the pages: 1536 sequences / "
                         "(DP 12 x MBS 2) = 64)")
    return ap.parse_args()


# ---------------------------------------------------------------- clocks

class ClockSampler:
    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        self.out = open(self.path, "w")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            self.out.close()
            os.unlink(self.path)
            self.path = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if self.proc is None or self.path is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- our arm

class Step:
    """Device buffers of one step and the launch sequence, with an event pair
    around every launch (on the launching stream)."""

    def __init__(self, wl, dev, n_sets=3):
        import torch
        import fp8_block_scaled_13_b200 as fp8
        from fp8_block_scaled_13_b200.dp import MainGrads
        self.fp8 = fp8
        self.torch = torch
        self.layers = wl.layers
        # rotating input sets: each set is larger than L2 in total
        self.sets = []
        for _ in range(n_sets):
            self.sets.append([(L.x.to(dev), L.w.to(dev), L.dy.to(dev)) for L in wl.layers])
        # outputs, allocated once and reused
        self.out = []
        for (x, w, dy) in self.sets[0]:
            xq = fp8.quant_act(x, "both")
            wq = fp8.quant_weight(w, transpose=True)
            dyq = fp8.quant_act(dy, "both")
            y = torch.empty((x.shape[0], w.shape[0]), dtype=torch.bfloat16, device=dev)
            dx = torch.empty_like(x)
            self.out.append((xq, wq, dyq, y, dx))
        # FP32 weight gradients of both layers in one buffer: every step adds
        # its dW into it (one micro-batch of gradient accumulation)
        self.grads = MainGrads([(w.shape[0], w.shape[1]) for (_, w, _) in self.sets[0]], device=dev)
        torch.cuda.synchronize()
        self.all_names = self.launch_names(True)

    def launch_names(self, weights):
        names = []
        for L in self.layers:
            if weights:
                names.append("%s.quant_weight" % L.name)
            names += ["%s.quant_x" % L.name, "%s.fprop" % L.name, "%s.quant_dy" % L.name,
                      "%s.dgrad_wgrad" % L.name]
        return names

    def run(self, set_idx, events=None, weights=True):
        """One micro-batch step.  The weights are quantized only when `weights`:
        within a gradient-accumulation window they do not change, so the first
        step's codes serve the whole window."""
        fp8 = self.fp8
        ev = iter(events) if events is not None else None

        def mark():
            if ev is not None:
                next(ev).record()

        for li, ((x, w, dy), (xq, wq, dyq, y, dx)) in enumerate(zip(self.sets[set_idx], self.out)):
            if weights:
                mark(); fp8.quant_weight(w, transpose=True, out=wq); mark()
            mark(); fp8.quant_act(x, "both", out=xq); mark()
            mark(); fp8.gemm_fprop(xq, wq, out=y); mark()
            mark(); fp8.quant_act(dy, "both", out=dyq); mark()
            mark(); fp8.gemm_dgrad_wgrad(dyq, wq, xq, dx=dx, dw=self.grads[li], accumulate=True); mark()

    def sync_grads(self, world):
        """End of a gradient-accumulation window: exchange the FP32 weight
        gradients across the data-parallel ranks (all-reduce, averaged), then
        clear them as the optimizer step would."""
        if world > 1:
            self.grads.all_reduce_(average=True)
        self.grads.zero_()


def _unit_costs(wl):
    """Algorithmic work per launch: FLOPs for the GEMMs, bytes for quantizers."""
    costs = {}
    for L in wl.layers:
        m, n, k = L.m, L.n, L.k
        costs["%s.quant_weight" % L.name] = ("bytes", n * k * 2 + 2 * n * k + (n // 128) * (k // 128))
        costs["%s.quant_x" % L.name] = ("bytes", m * k * 2 + 2 * m * k + 2 * m * k // 128)
        costs["%s.quant_dy" % L.name] = ("bytes", m * n * 2 + 2 * m * n + 2 * m * n // 128)
        costs["%s.fprop" % L.name] = ("flops", 2 * m * n * k)
        costs["%s.dgrad_wgrad" % L.name] = ("flops", 4 * m * n * k)
    return costs


def run_ours(args):
    import torch
    import torch.distributed as dist
    from fp8_block_scaled_13_b200 import inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    wl = inputs.attn_proj(seed=SEED + rank, m=M_TOKENS)
    step = Step(wl, dev)
    costs = _unit_costs(wl)
    gemm_flops = wl.gemm_flops()
    A = max(1, min(args.accum, args.steps))
    for i in range(args.warmup):
        step.run(i % len(step.sets), weights=(i % A == 0))
    torch.cuda.synchronize()
    status = step.fp8.device_status()
    if status != 0:
        raise RuntimeError("device status %d after warm-up" % status)

    # The timed steps run as CUDA graphs (kernel arguments, including the TMA
    # descriptors, are baked in), so the timed region holds device work only:
    # a graph of `accum` micro-batch steps is replayed, and after each window
    # the FP32 weight gradients are exchanged across the ranks (NCCL
    # all-reduce, outside the graph) and cleared; exactly K steps in all (a
    # shorter graph covers the remainder).  A separate graph with an event
    # pair around every launch gives the per-kernel breakdown; it is replayed
    # on its own because event nodes between kernels also cut the
    # programmatic (PDL) edges that let a kernel's prologue overlap its
    # predecessor's tail.
    K = args.steps
    windows = [A] * (K // A) + ([K % A] if K % A else [])
    K_inst = min(K, 100)
    inst_names = [step.launch_names(i % A == 0) for i in range(K_inst)]
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2 * len(nm))]
          for nm in inst_names]
    graphs = {}
    graph_inst = torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream()
    cap_stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap_stream):
        for n in sorted(set(windows)):
            graphs[n] = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graphs[n], stream=cap_stream):
                for i in range(n):
                    step.run(i % len(step.sets), weights=(i == 0))
        with torch.cuda.graph(graph_inst, stream=cap_stream):
            for i in range(K_inst):
                step.run(i % len(step.sets), ev[i], weights=(i % A == 0))
    torch.cuda.synchronize()
    for g in graphs.values():  # untimed first replays of the instantiated graphs
        g.replay()
    graph_inst.replay()
    step.sync_grads(world)
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_start.record()
        for n in windows:
            graphs[n].replay()
            step.sync_grads(world)
        t_end.record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    graph_inst.replay()
    torch.cuda.synchronize()
    status = step.fp8.device_status()
    if status != 0:
        raise RuntimeError("device status %d in the timed region" % status)
    clocks = clk.summary()

    total_ms = t_start.elapsed_time(t_end)
    per_launch = {name: [] for name in step.all_names}
    for i in range(K_inst):
        for j, name in enumerate(inst_names[i]):
            per_launch[name].append(ev[i][2 * j].elapsed_time(ev[i][2 * j + 1]))
    launches_timed = sum(n * len(step.launch_names(False)) + len(step.layers) for n in windows)
    ms_per_step = total_ms / K
    if world > 1:
        t = torch.tensor([ms_per_step], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_per_step = float(t.item())
    del graphs, graph_inst

    peaks, peak_kind = _peaks()
    fp8_peak_tf = 2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    value = gemm_flops * world / (ms_per_step * 1e-3) / 1e12

    gemm_ms = sum(statistics.mean(per_launch[n]) for n in step.all_names if costs[n][0] == "flops")
    gemm_tf = gemm_flops / (gemm_ms * 1e-3) / 1e12
    # quantizer bandwidth over every quantizer launch of the instrumented replay
    quant_ms = sum(sum(per_launch[n]) for n in step.all_names if costs[n][0] == "bytes")
    quant_bytes = sum(costs[n][1] * len(per_launch[n]) for n in step.all_names if costs[n][0] == "bytes")
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    breakdown = {}
    for n in step.all_names:
        kind, amount = costs[n]
        ms = statistics.mean(per_launch[n])
        rate = amount / (ms * 1e-3) / (1e12 if kind == "flops" else 1e9)
        breakdown[n] = {"ms": round(ms, 5), ("tflops" if kind == "flops" else "gbs"): round(rate, 1)}

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(wl, dev, K=min(K, 40), warmup=2, accum=A)
        if world > 1:
            t = torch.tensor([e2e["ms_per_step"]], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e["ms_per_step"] = float(t.item())
        e2e["value"] = round(gemm_flops * world / (e2e["ms_per_step"] * 1e-3) / 1e12, 2)

    ceiling = None
    if rank == 0 and not args.no_ceiling:
        ceiling = fp8_ceiling(wl, dev)

    bf16 = None
    if not args.no_bf16:
        bms = bf16_step_ms(step, min(K, 200))
        if world > 1:
            t = torch.tensor([bms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            bms = float(t.item())
        bf16 = {"ms_per_step": round(bms, 4),
                "tflops": round(gemm_flops / (bms * 1e-3) / 1e12, 1),
                "fp8_speedup": round(bms / ms_per_step, 3),
                "what": "same step in BF16 via torch.matmul (cuBLAS), no quantization; "
                        "fp8_speedup = BF16 step time / FP8 step time (quantizers included)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(value, 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": K,
            "warmup": args.warmup,
            "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e4m3",
            "data": "synthetic",
            "config": {
                "workload": WORKLOAD,
                "tokens_per_gpu": M_TOKENS, "hidden": 2048, "qkv_out": 3072, "o_out": 2048,
                "seed": SEED,
                "global_batch_tokens": M_TOKENS * world,
                "l2": "3 rotating input sets of 132 MB each (> 126 MB L2)",
                "parallelism": "dp%d (own batch per rank; FP32 dW all-reduce every %d steps)" % (world, A),
                "step": "per layer: quant_act(X), fprop, quant_act(dY), and one launch for "
                        "dgrad + wgrad (dW added into FP32 main grads); quant_weight once per "
                        "%d-step accumulation window (the weights do not change within it)" % A,
                "grad_exchange": "every %d steps: FP32 dW all-reduce across ranks (NCCL) and clear"
                                 % A,
            },
            "pct_fp8_peak": round(100.0 * value / world / fp8_peak_tf, 1),
            "roofline": {
                "bound": "tensor",
                "kernel": "gemm_block_scaled_kernel (fprop/dgrad/wgrad, FLOP-weighted)",
                "achieved": round(gemm_tf, 1),
                "peak": round(fp8_peak_tf, 1),
                "unit": "TFLOP/s",
                "frac": round(gemm_tf / fp8_peak_tf, 4),
                "peak_source": "%s: 2 x bf16_tflops_sustained (FP8 = 2 x BF16 nominal ratio)" % peak_kind,
                "traffic": GEMM_TRAFFIC_BYTES,
                "traffic_launch": "qkv.fprop (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            },
            "quantizers": {
                "bound": "hbm", "achieved": round(quant_gbs, 1), "unit": "GB/s",
                "peak": peaks["hbm_gbs"], "frac": round(quant_gbs / peaks["hbm_gbs"], 4),
                "traffic": QUANT_TRAFFIC_BYTES,
                "traffic_launch": "qkv.quant_x (ncu dram__bytes_read.sum + dram__bytes_write.sum)",
            },
            "kernels": breakdown,
            "gpu_launches": launches_timed,
            "clocks": clocks,
            "wall_ms_timed_region": round(total_ms, 3),
            "timing": "K steps as CUDA graphs of %d steps plus the gradient exchange between them "
                      "(device events around it all); per-kernel times from a separate replay of %d "
                      "steps with an event pair around every launch" % (A, K_inst),
        }
        if e2e is not None:
            line["e2e"] = {"value": e2e["value"], "unit": "TFLOP/s",
                           "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                           "ms_per_step": round(e2e["ms_per_step"], 3)}
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if bf16 is not None:
            line["bf16_comparison"] = bf16
            line["mfu_accounting"] = mfu_accounting(value / world, bf16["tflops"], peaks)
        if ceiling is not None:
            if "tflops_step_shapes" in ceiling:
                ceiling["gemm_vs_library_same_shapes"] = round(gemm_tf / ceiling["tflops_step_shapes"], 3)
            line["fp8_library_ceiling"] = ceiling
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def bf16_step_ms(step, K):
    """The same linear step in BF16 through cuBLAS (torch.matmul): per layer
    Y = X W^T, dX = dY W, dW = dY^T X, on the same rotating device input sets,
    K steps captured in one CUDA graph and timed with device events.  This is
    the FP8-vs-BF16 comparison of the pages' throughput claim, taken at the
    level of the linear layer."""
    import torch
    outs = []
    for (x, w, dy) in step.sets[0]:
        outs.append((torch.empty((x.shape[0], w.shape[0]), dtype=torch.bfloat16, device=x.device),
                     torch.empty_like(x), torch.empty_like(w)))

    def one(i):
        for (x, w, dy), (y, dx, dw) in zip(step.sets[i % len(step.sets)], outs):
            torch.matmul(x, w.t(), out=y)
            torch.matmul(dy, w, out=dx)
            torch.matmul(dy.t(), x, out=dw)

    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True, external=True)
    t1 = torch.cuda.Event(enable_timing=True, external=True)
    g = torch.cuda.CUDAGraph()
    cs = torch.cuda.Stream()
    cs.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cs):
        with torch.cuda.graph(g, stream=cs):
            t0.record()
            for i in range(K):
                one(i)
            t1.record()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / K
    del g
    return ms


def mfu_accounting(fp8_tflops, bf16_tflops, peaks):
    """Mixed-precision MFU bookkeeping with the pages' weighting: 72 % of a
    step's FLOPs in FP8 linear layers, 28 % in BF16.  The effective peak is the
    time-weighted (harmonic) mean P_eff = (0.72/P_fp8 + 0.28/P_bf16)^-1; the
    projected throughput combines the measured FP8 linear-layer rate with the
    measured BF16 cuBLAS rate on the same shapes for the BF16 share."""
    f8, bf = 0.72, 0.28
    nominal = {"fp8": 4500.0, "bf16": 2250.0}
    measured = {"fp8": 2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "bf16": peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])}
    proj = 1.0 / (f8 / fp8_tflops + bf / bf16_tflops)
    out = {"fp8_share": f8, "bf16_share": bf,
           "fp8_tflops_measured": round(fp8_tflops, 1), "bf16_tflops_measured": round(bf16_tflops, 1),
           "projected_tflops": round(proj, 1)}
    for name, pk in (("nominal", nominal), ("measured", measured)):
        peff = 1.0 / (f8 / pk["fp8"] + bf / pk["bf16"])
        out["p_eff_%s" % name] = round(peff, 1)
        out["mfu_vs_%s" % name] = round(proj / peff, 4)
    return out


def fp8_ceiling(wl, dev):
    """Library FP8 tensor-core throughput on this GPU, for context: cuBLASLt's
    MXFP8 GEMM (E4M3 operands, UE8M0 scales per 1x32 block, BF16 out) through
    torch's scaled_mm, at 8192^3 and at the six GEMM shapes of the step.  Not
    the same scaling granularity as the path (1x128 / 128x128), so it is a
    ceiling estimate, not a comparison arm.  None if unavailable."""
    import torch
    import torch.nn.functional as F
    if not hasattr(F, "scaled_mm") or not hasattr(torch, "float8_e8m0fnu"):
        return None

    def rup(a, b):
        return (a + b - 1) // b * b

    def timed(m, n, k, reps=20):
        # random operands: constant ones draw less power and run at clocks a
        # real GEMM does not keep (measured: 4.0 vs 2.6 PF/s at 8192^3)
        g = torch.Generator(device=dev).manual_seed(7)
        a = (torch.randn((m, k), device=dev, generator=g) * 4).to(torch.float8_e4m3fn)
        b = (torch.randn((n, k), device=dev, generator=g) * 4).to(torch.float8_e4m3fn)
        sa = torch.full((rup(m, 128) * rup(k // 32, 4),), 127, dtype=torch.uint8,
                        device=dev).view(torch.float8_e8m0fnu)
        sb = torch.full((rup(n, 128) * rup(k // 32, 4),), 127, dtype=torch.uint8,
                        device=dev).view(torch.float8_e8m0fnu)

        def f():
            return F.scaled_mm(a, b.t(), sa, F.ScalingType.BlockWise1x32, sb,
                               F.ScalingType.BlockWise1x32,
                               swizzle_a=F.SwizzleType.SWIZZLE_32_4_4,
                               swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                               output_dtype=torch.bfloat16)
        for _ in range(3):
            f()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(reps)]
        for s0, s1 in ev:
            s0.record(); f(); s1.record()
        torch.cuda.synchronize()
        ms = sorted(s0.elapsed_time(s1) for s0, s1 in ev)[reps // 2]
        return ms

    try:
        ms = timed(8192, 8192, 8192)
        peak = 2.0 * 8192 ** 3 / (ms * 1e-3) / 1e12
        tot_ms, tot_flops = 0.0, 0
        for L in wl.layers:
            for (m, n, k) in ((L.m, L.n, L.k), (L.m, L.k, L.n), (L.n, L.k, L.m)):
                tot_ms += timed(m, n, k)
                tot_flops += 2 * m * n * k
        return {"source": "cuBLASLt MXFP8 via torch scaled_mm (1x32 UE8M0 scales, BF16 out)",
                "tflops_8192cube": round(peak, 1),
                "tflops_step_shapes": round(tot_flops / (tot_ms * 1e-3) / 1e12, 1)}
    except Exception as e:  # noqa: BLE001  (library path missing on this build)
        return {"unavailable": str(e).splitlines()[0][:160]}


def run_e2e(wl, dev, K, warmup, accum):
    """Same step through the public API with pinned host inputs/outputs, inside
    the timed region: every step copies X and dY in (and, at the start of each
    `accum`-step accumulation window, W, which is then quantized once for the
    window), runs forward and backward (dW added into the FP32 main grads), and
    copies Y and dX back; the main grads go back when they are complete, at
    the end of each window (and of the run), as an optimizer would read them.
    The copies are pipelined across steps the way a training loop would: step
    i+1's inputs go up on a copy stream while step i computes, and step i's
    results come down on another while step i+1 computes (double-buffered
    inputs and outputs, ordered by events)."""
    import torch
    import fp8_block_scaled_13_b200 as fp8
    from fp8_block_scaled_13_b200.dp import MainGrads

    nbuf = 2
    host_w = [L.w.pin_memory() for L in wl.layers]
    host_in = [[(L.x.pin_memory(), L.dy.pin_memory()) for L in wl.layers] for _ in range(nbuf)]
    host_out = [[(torch.empty((L.m, L.n), dtype=torch.bfloat16).pin_memory(),
                  torch.empty((L.m, L.k), dtype=torch.bfloat16).pin_memory()) for L in wl.layers]
                for _ in range(nbuf)]
    host_dw = [torch.empty((L.n, L.k), dtype=torch.float32).pin_memory() for L in wl.layers]
    dev_w = [torch.empty_like(w, device=dev) for w in host_w]
    dev_in = [[(torch.empty_like(x, device=dev), torch.empty_like(dy, device=dev))
               for (x, dy) in host_in[0]] for _ in range(nbuf)]
    wq = [None] * len(wl.layers)
    results = [None] * nbuf   # device outputs (Y, dX) of the step that used buffer b
    grads = MainGrads([(L.n, L.k) for L in wl.layers], device=dev)
    bytes_w = sum(t.numel() * t.element_size() for t in host_w)
    bytes_in = sum(t.numel() * t.element_size() for tup in host_in[0] for t in tup)
    bytes_out = sum(t.numel() * t.element_size() for tup in host_out[0] for t in tup)
    bytes_dw = sum(t.numel() * t.element_size() for t in host_dw)
    comp = torch.cuda.current_stream()
    up = torch.cuda.Stream()
    down = torch.cuda.Stream()
    ev_up = [torch.cuda.Event() for _ in range(nbuf)]      # inputs of buffer b are on the device
    ev_done = [torch.cuda.Event() for _ in range(nbuf)]    # compute on buffer b finished
    ev_down = [torch.cuda.Event() for _ in range(nbuf)]    # results of buffer b are on the host
    ev_dw_down = torch.cuda.Event()                        # the last window's dW is on the host

    def upload(i):
        b = i % nbuf
        with torch.cuda.stream(up):
            up.wait_event(ev_done[b])   # the previous use of these device buffers is over
            if i % accum == 0:
                up.wait_event(ev_done[(i - 1) % nbuf])   # the last user of the old weights
                for hw, w in zip(host_w, dev_w):
                    w.copy_(hw, non_blocking=True)
            for (hx, hdy), (x, dy) in zip(host_in[b], dev_in[b]):
                x.copy_(hx, non_blocking=True)
                dy.copy_(hdy, non_blocking=True)
            ev_up[b].record(up)

    def compute(i):
        b = i % nbuf
        comp.wait_event(ev_up[b])
        comp.wait_event(ev_down[b])   # the previous results of buffer b went down
        if i % accum == 0:
            comp.wait_event(ev_dw_down)   # the previous window's dW went down
            grads.zero_()
        outs = []
        for li, (x, dy) in enumerate(dev_in[b]):
            if i % accum == 0:
                y, xq, wq[li] = fp8.linear_forward(x, dev_w[li])
            else:
                y, xq, _ = fp8.linear_forward(x, wq=wq[li])
            dx, _ = fp8.linear_backward(dy, xq, wq[li], main_grad=grads[li])
            y.record_stream(down)
            dx.record_stream(down)
            outs.append((y, dx))
        results[b] = outs
        ev_done[b].record(comp)

    def download(i, last):
        b = i % nbuf
        with torch.cuda.stream(down):
            down.wait_event(ev_done[b])
            for li, ((hy, hdx), (y, dx)) in enumerate(zip(host_out[b], results[b])):
                hy.copy_(y, non_blocking=True)
                hdx.copy_(dx, non_blocking=True)
            ev_down[b].record(down)
            if i % accum == accum - 1 or last:
                for hdw, g in zip(host_dw, grads.views):
                    hdw.copy_(g, non_blocking=True)
                ev_dw_down.record(down)

    def run(n):
        upload(0)
        for i in range(n):
            if i + 1 < n:
                upload(i + 1)
            compute(i)
            download(i, i == n - 1)
        torch.cuda.synchronize()

    run(warmup)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    s.record()
    run(K)
    e.record()
    torch.cuda.synchronize()
    windows = (K + accum - 1) // accum
    return {"ms_per_step": s.elapsed_time(e) / K,
            "h2d": int(bytes_in + bytes_w * windows / K),
            "d2h": int(bytes_out + bytes_dw * windows / K)}


# ---------------------------------------------------------------- CPU oracle

def _oracle_sample(wl, rows_per_gemm):
    """The hot path on a bounded sample, through the CPU oracle: for every
    layer, `rows_per_gemm` output rows of fprop, dgrad and wgrad, including the
    quantization those rows need.  Returns the sampled GEMM FLOPs."""
    import numpy as np
    import oracle

    flops = 0
    for L in wl.layers:
        m, n, k = L.m, L.n, L.k
        r = rows_per_gemm
        rows = np.linspace(0, m - 1, r).astype(np.int64)
        oracle.linear_fprop(L.x[rows], L.w)
        oracle.linear_dgrad(L.dy[rows], L.w)
        cols = np.linspace(0, n - 1, r).astype(np.int64)
        oracle.linear_wgrad(L.dy[:, cols].contiguous(), L.x)
        flops += 3 * 2 * r * n * k
    return flops


def cpu_baseline(wl, min_s=10.0):
    """Times the oracle on a sample of the workload that takes at least `min_s`
    seconds: the number of sampled output rows doubles until one sample run
    lasts that long (the last run is the reported one, so it lasts between
    `min_s` and about twice that)."""
    n_cores = len(os.sched_getaffinity(0))
    rows = 16
    while True:
        t0 = time.perf_counter()
        f = _oracle_sample(wl, rows)
        dt = time.perf_counter() - t0
        if dt >= min_s or rows >= 8192:
            break
        rows *= 2
    return {"value": round(f / dt / 1e12, 6), "unit": "TFLOP/s", "cores": n_cores,
            "kind": "oracle",
            "sample": "%d output rows of each of the 6 GEMMs (fprop/dgrad/wgrad x 2 layers) "
                      "with the quantization they need, FP64 C oracle, %.1f s" % (rows, dt)}


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on a bounded sample of the
    same workload per step; rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from fp8_block_scaled_13_b200 import inputs
    wl = inputs.attn_proj(seed=SEED, m=M_TOKENS)
    rows = 8
    for _ in range(args.warmup):
        _oracle_sample(wl, rows)
    t0 = time.perf_counter()
    flops = 0
    for _ in range(args.steps):
        flops += _oracle_sample(wl, rows)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    n_cores = len(os.sched_getaffinity(0))
    sample = ("%d output rows of each of the 6 GEMMs per step (fprop/dgrad/wgrad x 2 layers) "
              "with the quantization they need, FP64 C oracle" % rows)
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "tokens_per_gpu": M_TOKENS, "hidden": 2048,
                   "qkv_out": 3072, "o_out": 2048, "seed": SEED},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": n_cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def main():
    args = _parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
