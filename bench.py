"""Benchmark of the block-scaled FP8 linear layer hot path on B200.

A step is one forward + backward pass of every linear layer of a workload over
one batch of M tokens (inputs resident in HBM).  For each layer:
  quant_act(X, both), fprop, quant_act(dY, both), and one launch computing
  dgrad and wgrad (dW added into FP32 main grads); quant_weight(W) (+
  transposed codes) runs once per gradient-accumulation window of --accum
  steps, since the weights only change at the optimizer step.
value = GEMM FLOPs of the step (2*M*N*K per GEMM, three GEMMs per layer)
divided by the device time of the whole step (quantizers included).

The default workload is the full hidden-2048 / FFN-6144 transformer block
(QKV 2048->3072, O 2048->2048, gate+up 2048->12288, down 6144->2048) at
M = 32768 tokens, the largest single-GPU configuration; a sweep of the other
configurations (attention projections, SwiGLU gate+up, heavy-tailed MLP down,
the full block at M = 4096, 8000, 16384) follows as summaries in the same
JSON line.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                       [--tokens M] [--accum A] [--impl ours|reference]
                       [--no-sweep] [--no-e2e] [--no-cpu-baseline] [--no-bf16]
                       [--no-ceiling]
N > 1: every rank runs its own batch (data parallel, weak scaling) and every A
steps the ranks all-reduce the FP32 weight gradients (NCCL).  Launched without
torchrun, bench.py starts the N ranks itself (torch.distributed.run).
"""
from __future__ import annotations

import argparse
import json
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "FP8 block-scaled GEMM TFLOP/s (fprop/dgrad/wgrad) and % of B200 FP8 peak"

# workload -> (default tokens, seed, shapes for the config record)
WORKLOADS = {
    "full_block": (32768, 4, "hidden 2048, FFN 6144: QKV 2048->3072, O 2048->2048, "
                             "gate+up 2048->12288, down 6144->2048"),
    "attn_proj": (8192, 1, "hidden 2048: QKV 2048->3072, O 2048->2048 (shared X)"),
    "swiglu_gate_up": (16384, 2, "gate+up 2048->12288, 8 channels of X x50"),
    "mlp_down_heavy": (16384, 3, "down 6144->2048, Student-t(3) X, Laplace dY, zero groups"),
}
SWEEP = [("attn_proj", 8192), ("swiglu_gate_up", 16384), ("mlp_down_heavy", 16384),
         ("full_block", 4096), ("full_block", 8000), ("full_block", 16384)]
# tokens per gradient-accumulation window: the pages' 1536 sequences /
# (DP 12 x MBS 2) = 64 micro-batches of 2 x 4096 tokens
WINDOW_TOKENS = 64 * 8192
L2_BYTES = 126 * 1024 * 1024
SPEC_FP8_TFLOPS = 4500.0     # B200 dense FP8 tensor-core peak (spec)
SPEC_BF16_TFLOPS = 2250.0
SPEC_HBM_GBS = 8000.0
SPEC_SM_MHZ = 1965.0         # B200 maximum SM clock, at which the spec peak is quoted
LOADED_WATTS = 500.0         # board power above which a clock sample counts as under load

# dram__bytes_read.sum + dram__bytes_write.sum of every launch of one step of
# the default workload (full block, 32768 tokens), from a one-pass ncu capture
# of the current kernels:
#   ncu --clock-control none --metrics gpu__time_duration.sum,dram__bytes_read.sum,
#       dram__bytes_write.sum -c 200 --csv python bench.py --steps 2 --warmup 1
#       --accum 2 --no-sweep --no-e2e --no-cpu-baseline --no-ceiling --no-bf16
# (serialised launches: each one starts with its inputs in DRAM, and what it
# writes last may still sit in L2 when it ends).  To be emptied whenever a
# kernel changes, until it is captured again.
TRAFFIC_WORKLOAD = "full_block_m32768"
TRAFFIC_BYTES = {
    "qkv.quant_weight": 12_600_000, "qkv.quant_x": 209_600_000, "qkv.fprop": 221_700_000,
    "qkv.quant_dy": 345_000_000, "qkv.dgrad_wgrad": 497_300_000,
    "o_proj.quant_weight": 8_400_000, "o_proj.quant_x": 213_000_000, "o_proj.fprop": 156_300_000,
    "o_proj.quant_dy": 209_400_000, "o_proj.dgrad_wgrad": 328_300_000,
    "gate_up.quant_weight": 50_900_000, "gate_up.quant_x": 209_900_000, "gate_up.fprop": 883_800_000,
    "gate_up.quant_dy": 1_559_100_000, "gate_up.dgrad_wgrad": 1_762_200_000,
    "down.quant_weight": 25_200_000, "down.quant_x": 750_900_000, "down.fprop": 325_300_000,
    "down.quant_dy": 209_200_000, "down.dgrad_wgrad": 994_600_000,
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def _parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="full_block")
    ap.add_argument("--tokens", dest="m", type=int, default=None,
                    help="tokens per GPU per step (M)")
    ap.add_argument("--accum", type=int, default=None,
                    help="steps per gradient exchange (default: a window of 64 x 8192 tokens)")
    ap.add_argument("--no-sweep", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-ceiling", action="store_true")
    ap.add_argument("--no-bf16", action="store_true")
    args = ap.parse_args(argv)
    if args.m is None:
        args.m = WORKLOADS[args.workload][0]
    if args.accum is None:
        args.accum = max(1, WINDOW_TOKENS // args.m)
    if args.gpus < 1 or args.steps < 1 or args.warmup < 0 or args.m < 1:
        ap.error("--gpus, --steps, --tokens must be >= 1 and --warmup >= 0")
    return args


def make_workload(name: str, m: int, seed_offset: int = 0):
    from fp8_block_scaled_13_b200 import inputs
    seed = WORKLOADS[name][1] + seed_offset
    return inputs.WORKLOADS[name](seed=seed, m=m)


def workload_tag(name: str, m: int) -> str:
    return "%s_m%d" % (name, m)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of the SM clock, utilisation and throttle reasons
    while the context is open; the summary takes the median clock over the
    samples taken under load (utilisation >= 50 %)."""

    def __init__(self, gpu: str, period_ms: int = 50):
        self.gpu = gpu
        self.period = period_ms
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        self.out = open(self.path, "w")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + q,
                 "--format=csv,noheader,nounits", "-lms", str(self.period)],
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
        return summarize_clocks(rows)


def smi_id(device_index: int) -> str:
    """nvidia-smi's name for a CUDA device: its UUID (device indexes differ
    between CUDA and nvidia-smi when CUDA_VISIBLE_DEVICES is set)."""
    try:
        import torch
        u = str(torch.cuda.get_device_properties(device_index).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:  # noqa: BLE001  (older torch without a uuid field)
        return str(device_index)


def _num(s):
    try:
        return float(s)
    except ValueError:
        return None


def summarize_clocks(rows):
    """rows: nvidia-smi fields index, clocks.sm, clocks.max.sm, power.draw,
    utilization.gpu, hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown,
    sw_power_cap.  A sample is under load when the utilisation reads >= 50 %
    or the board draws >= LOADED_WATTS (the utilisation counter averages over
    a longer window than the sampling period and lags behind a short run).
    Median SM clock over the loaded samples (all samples if none is loaded);
    every throttle reason seen Active in a loaded sample."""
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
    loaded = [r for r in rows if (_num(r[4]) or 0.0) >= 50.0 or (_num(r[3]) or 0.0) >= LOADED_WATTS]
    use = loaded or rows
    sm = [v for v in (_num(r[1]) for r in use) if v is not None]
    mx = [v for v in (_num(r[2]) for r in rows) if v is not None]
    pw = [v for v in (_num(r[3]) for r in use) if v is not None]
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    reasons = sorted({names[i] for r in use for i in range(4) if r[5 + i] == "Active"})
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None,
            "power_w": round(statistics.median(pw), 1) if pw else None,
            "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded)}


# ---------------------------------------------------------------- our arm

class Step:
    """Device buffers of one step and the launch sequence, with an optional
    event pair around every launch (on the launching stream)."""

    def __init__(self, wl, dev, n_sets):
        import torch
        import fp8_block_scaled_13_b200 as fp8
        from fp8_block_scaled_13_b200.dp import MainGrads
        self.fp8 = fp8
        self.torch = torch
        self.layers = wl.layers
        # input sets: rotated so that every step's inputs come from HBM
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
        # FP32 weight gradients of all layers in one buffer: every step adds
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
        """One step.  The weights are quantized only when `weights`: within a
        gradient-accumulation window they do not change, so the first step's
        codes serve the whole window."""
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


def input_set_bytes(wl) -> int:
    return sum(t.numel() * t.element_size() for L in wl.layers for t in (L.x, L.w, L.dy))


def n_input_sets(wl) -> int:
    """Enough rotating input sets that the inputs a step reads were last read
    at least three L2 capacities of traffic ago (one set when a single set
    already is)."""
    per = input_set_bytes(wl)
    return max(1, min(3, -(-3 * L2_BYTES // per)))


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


def measure(wl, dev, world, K, warmup, accum, gpu, inst_steps=100):
    """Times K steps of the workload on the device (CUDA graphs of `accum`
    steps, the gradient exchange between them) and, separately, per-launch
    times from an instrumented replay of `inst_steps` steps (long enough for
    the clock samples taken over both to catch the GPU under load).  Returns
    the raw measurements."""
    import torch
    import torch.distributed as dist

    n_sets = n_input_sets(wl)
    step = Step(wl, dev, n_sets)
    A = max(1, min(accum, K))
    for i in range(warmup):
        step.run(i % n_sets, weights=(i % A == 0))
    torch.cuda.synchronize()
    status = step.fp8.device_status()
    if status != 0:
        raise RuntimeError("device status %d after warm-up" % status)

    # The timed steps run as CUDA graphs (kernel arguments, including the TMA
    # descriptors, are baked in), so the timed region holds device work only:
    # a graph of `accum` steps is replayed, and after each window the FP32
    # weight gradients are exchanged across the ranks (NCCL all-reduce,
    # outside the graph) and cleared; exactly K steps in all (a shorter graph
    # covers the remainder).  A separate graph with an event pair around every
    # launch gives the per-kernel breakdown; it is replayed on its own because
    # event nodes between kernels also cut the programmatic (PDL) edges that
    # let a kernel's prologue overlap its predecessor's tail.
    windows = [A] * (K // A) + ([K % A] if K % A else [])
    K_inst = inst_steps
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
                    step.run(i % n_sets, weights=(i == 0))
        with torch.cuda.graph(graph_inst, stream=cap_stream):
            for i in range(K_inst):
                step.run(i % n_sets, ev[i], weights=(i % A == 0))
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
    with ClockSampler(gpu) as clk:
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
    return {"step": step, "ms_per_step": ms_per_step, "total_ms": total_ms, "accum": A,
            "per_launch": per_launch, "clocks": clk.summary(), "launches_timed": launches_timed,
            "inst_steps": K_inst, "n_sets": n_sets}


def summarize(wl, res, peaks, peak_kind, world, wl_tag=None):
    """value, GEMM roofline, quantizer roofline and per-kernel breakdown."""
    costs = _unit_costs(wl)
    gemm_flops = wl.gemm_flops()
    names = res["step"].all_names
    pl = res["per_launch"]
    value = gemm_flops * world / (res["ms_per_step"] * 1e-3) / 1e12
    gemm_ms = sum(statistics.mean(pl[n]) for n in names if costs[n][0] == "flops")
    gemm_tf = gemm_flops / (gemm_ms * 1e-3) / 1e12
    # quantizer bandwidth over every quantizer launch of the instrumented replay
    quant_ms = sum(sum(pl[n]) for n in names if costs[n][0] == "bytes")
    quant_bytes = sum(costs[n][1] * len(pl[n]) for n in names if costs[n][0] == "bytes")
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9
    act_names = [n for n in names if costs[n][0] == "bytes" and not n.endswith("quant_weight")]
    act_ms = sum(sum(pl[n]) for n in act_names)
    act_gbs = sum(costs[n][1] * len(pl[n]) for n in act_names) / (act_ms * 1e-3) / 1e9
    traffic = TRAFFIC_BYTES if wl_tag == TRAFFIC_WORKLOAD else {}
    breakdown = {}
    for n in names:
        kind, amount = costs[n]
        ms = statistics.mean(pl[n])
        rate = amount / (ms * 1e-3) / (1e12 if kind == "flops" else 1e9)
        breakdown[n] = {"ms": round(ms, 5), ("tflops" if kind == "flops" else "gbs"): round(rate, 1)}
        if n in traffic:
            breakdown[n]["dram_bytes"] = traffic[n]
            if kind == "bytes":
                breakdown[n]["algorithmic_bytes"] = amount

    def mean_traffic(which):
        sel = [n for n in names if costs[n][0] == which]
        if not traffic or any(n not in traffic for n in sel):
            return None
        return int(sum(traffic[n] for n in sel) / len(sel))
    burst = 2.0 * peaks["bf16_tflops"]
    sustained = 2.0 * peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    peak, regime = gemm_peak(res["clocks"], burst, sustained)
    clk = res["clocks"].get("sm_mhz")
    per_step_ms = {"gemm": gemm_ms,
                   "quant_act": act_ms / res["inst_steps"],
                   "quant_weight": (quant_ms - act_ms) / res["inst_steps"]}
    roofline = {
        "bound": "tensor",
        "kernel": "gemm_block_scaled_kernel (every GEMM launch of the step, FLOP-weighted)",
        "achieved": round(gemm_tf, 1),
        "peak": round(peak, 1),
        "unit": "TFLOP/s",
        "frac": round(gemm_tf / peak, 4),
        "peak_source": "%s: 2 x bf16_tflops%s (%s cuBLAS BF16 GEMM) x the nominal FP8:BF16 ratio "
                       "of 2, of %s; %s" % (peak_kind, "_sustained" if regime == "sustained" else "",
                                            regime, peak_kind, REGIME_RULE),
        "frac_vs_burst": round(gemm_tf / burst, 4),
        "frac_vs_sustained": round(gemm_tf / sustained, 4),
        "frac_vs_spec": round(gemm_tf / SPEC_FP8_TFLOPS, 4),
        "spec_peak": SPEC_FP8_TFLOPS,
        "frac_vs_spec_at_clock": (round(gemm_tf / (SPEC_FP8_TFLOPS * clk / SPEC_SM_MHZ), 4)
                                  if clk else None),
        "traffic": mean_traffic("flops"),
        "traffic_what": "DRAM bytes read + written per GEMM launch, averaged over the step's GEMM "
                        "launches (per launch in `kernels`), from a one-pass ncu capture",
    }
    quant = {
        "bound": "hbm", "achieved": round(quant_gbs, 1), "unit": "GB/s",
        "peak": peaks["hbm_gbs"], "frac": round(quant_gbs / peaks["hbm_gbs"], 4),
        "peak_source": "%s: hbm_gbs (STREAM-style copy); of %s" % (peak_kind, peak_kind),
        "frac_vs_spec": round(quant_gbs / SPEC_HBM_GBS, 4), "spec_peak": SPEC_HBM_GBS,
        "activations_only": {"achieved": round(act_gbs, 1),
                             "frac": round(act_gbs / peaks["hbm_gbs"], 4)},
        "traffic": mean_traffic("bytes"),
        "what": "every quantizer launch of the instrumented replay, algorithmic bytes over "
                "per-launch event time (each launch timed on its own, without the overlap "
                "with its neighbours that the timed graphs have)",
    }
    return {"value": value, "gemm_tf": gemm_tf, "roofline": roofline, "quantizers": quant,
            "kernels": breakdown, "gemm_flops": gemm_flops,
            "time_split_ms_per_step": {k: round(v, 4) for k, v in per_step_ms.items()},
            "pct_of_spec_fp8_peak": round(100.0 * value / world / SPEC_FP8_TFLOPS, 1)}


REGIME_RULE = ("the sustained peak applies when the clock record shows sw_power_cap and a "
               "median SM clock under 0.9 x max (a long, power-capped run), the burst peak "
               "otherwise; frac_vs_spec_at_clock scales the 4.5 PF/s spec to the median clock")


def gemm_peak(clocks, burst, sustained):
    """The FP8 tensor peak the GEMM rate is compared with, and its regime."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = ("sw_power_cap" in clocks.get("reasons", []) and mhz is not None and mx
              and mhz < 0.9 * mx)
    return (sustained, "sustained") if capped else (burst, "burst")


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("bench.py: --gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    if world > 1:
        os.environ.setdefault("NCCL_DEBUG", "INFO")
        if torch.cuda.device_count() < world:
            raise SystemExit("bench.py: %d ranks but %d visible GPUs" % (world, torch.cuda.device_count()))
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_kind = _peaks()

    wl = make_workload(args.workload, args.m, seed_offset=rank)
    set_bytes = input_set_bytes(wl)
    res = measure(wl, dev, world, args.steps, args.warmup, args.accum, smi_id(local))
    sm = summarize(wl, res, peaks, peak_kind, world, workload_tag(args.workload, args.m))
    step = res["step"]
    A = res["accum"]
    gemm_flops = sm["gemm_flops"]

    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(wl, dev, K=min(args.steps, e2e_steps(wl)), warmup=2, accum=A)
        if world > 1:
            t = torch.tensor([e2e["ms_per_step"]], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e2e["ms_per_step"] = float(t.item())
        e2e["value"] = round(gemm_flops * world / (e2e["ms_per_step"] * 1e-3) / 1e12, 2)

    ceiling = None
    if rank == 0 and not args.no_ceiling:
        ceiling = fp8_ceiling(wl, dev)
        if ceiling is not None and world == 1:
            ceiling["sustained_same_codes"] = gemm_sustained(step, dev, smi_id(local))

    bf16 = None
    if not args.no_bf16:
        bms = bf16_step_ms(step, min(args.steps, 50))
        if world > 1:
            t = torch.tensor([bms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            bms = float(t.item())
        bf16 = bf16_summary(bms, res["ms_per_step"], gemm_flops)
    del step, res["step"]
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)
    del wl

    sweep = None
    if world == 1 and not args.no_sweep:
        sweep = run_sweep(args, dev, peaks, peak_kind)

    if rank == 0:
        line = {
            "metric": METRIC,
            "value": round(sm["value"], 2),
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": round(res["ms_per_step"], 4),
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e4m3",
            "data": "synthetic",
            "config": {
                "workload": workload_tag(args.workload, args.m),
                "layers": WORKLOADS[args.workload][2],
                "tokens_per_gpu": args.m,
                "seed": WORKLOADS[args.workload][1],
                "global_batch_tokens": args.m * world,
                "gemm_flops_per_step": gemm_flops,
                "l2": "%d input set(s) of %.0f MB rotated: the inputs a step reads were last read "
                      "at least 3 x 126 MB (L2) of inputs earlier" % (res["n_sets"], set_bytes / 1e6),
                "parallelism": "dp%d (own batch per rank; FP32 dW all-reduce every %d steps)" % (world, A),
                "step": "per layer: quant_act(X), fprop, quant_act(dY), and one launch for "
                        "dgrad + wgrad (dW added into FP32 main grads); quant_weight once per "
                        "%d-step accumulation window (the weights do not change within it)" % A,
                "grad_exchange": "every %d steps: FP32 dW all-reduce across ranks (NCCL) and clear" % A,
            },
            "pct_of_spec_fp8_peak": sm["pct_of_spec_fp8_peak"],
            "roofline": sm["roofline"],
            "quantizers": sm["quantizers"],
            "time_split_ms_per_step": sm["time_split_ms_per_step"],
            "kernels": sm["kernels"],
            "gpu_launches": res["launches_timed"],
            "clocks": res["clocks"],
            "wall_ms_timed_region": round(res["total_ms"], 3),
            "timing": "K steps as CUDA graphs of %d steps plus the gradient exchange between them "
                      "(device events around it all); per-kernel times from a separate replay of %d "
                      "steps with an event pair around every launch; clocks sampled over both"
                      % (A, res["inst_steps"]),
        }
        if e2e is not None:
            line["e2e"] = {"value": e2e["value"], "unit": "TFLOP/s",
                           "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                           "ms_per_step": round(e2e["ms_per_step"], 3), "steps": e2e["steps"]}
        if cpu is not None:
            line["cpu_baseline"] = cpu
        if bf16 is not None:
            line["bf16_comparison"] = bf16
            line["mfu_accounting"] = mfu_accounting(sm["value"] / world, bf16["tflops"], peaks)
        if ceiling is not None:
            if "tflops_step_shapes" in ceiling:
                ceiling["gemm_vs_library_same_shapes"] = round(sm["gemm_tf"] / ceiling["tflops_step_shapes"], 3)
            line["fp8_library_ceiling"] = ceiling
        if sweep is not None:
            line["sweep"] = sweep
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def e2e_steps(wl) -> int:
    """Steps of the end-to-end measure: about 40 at the attention-projection
    size, fewer for larger workloads (their steps are PCIe-bound and long),
    but at least 20: the first step's upload and the last step's download
    cannot overlap anything, and over 6 steps of the full block they added
    ~14 ms to every ~50 ms step."""
    per = input_set_bytes(wl)
    return max(20, min(40, int(40 * 2.7e8 / per)))


def bf16_summary(bms, fp8_ms, gemm_flops):
    return {"ms_per_step": round(bms, 4),
            "tflops": round(gemm_flops / (bms * 1e-3) / 1e12, 1),
            "fp8_speedup": round(bms / fp8_ms, 3),
            "what": "same step in BF16 via torch.matmul (cuBLAS), no quantization; "
                    "fp8_speedup = BF16 step time / FP8 step time (quantizers included)"}


def run_sweep(args, dev, peaks, peak_kind):
    """Short measurements of the other configurations (N = 1): the step rate,
    the GEMM and quantizer rooflines, the FP8-vs-BF16 ratio, MFU accounting,
    the end-to-end rate and the oracle baseline for each."""
    import torch
    out = {}
    K = max(3, min(args.steps, 20))
    for name, m in SWEEP:
        if name == args.workload and m == args.m:
            continue
        wl = make_workload(name, m)
        A = max(1, WINDOW_TOKENS // m)
        res = measure(wl, dev, 1, K, max(3, min(args.warmup, 5)), A, smi_id(dev.index))
        sm = summarize(wl, res, peaks, peak_kind, 1, workload_tag(name, m))
        entry = {"ms_per_step": round(res["ms_per_step"], 4), "value": round(sm["value"], 1),
                 "unit": "TFLOP/s", "steps": K, "accum": A,
                 "gemm_tflops": round(sm["gemm_tf"], 1),
                 "gemm_frac": sm["roofline"]["frac"],
                 "gemm_frac_vs_spec": sm["roofline"]["frac_vs_spec"],
                 "quant_gbs": sm["quantizers"]["achieved"],
                 "quant_frac": sm["quantizers"]["frac"],
                 "quant_act_frac": sm["quantizers"]["activations_only"]["frac"],
                 "time_split_ms_per_step": sm["time_split_ms_per_step"],
                 "kernels": sm["kernels"], "clocks": res["clocks"]}
        if not args.no_bf16:
            bms = bf16_step_ms(res["step"], K)
            entry["bf16_comparison"] = bf16_summary(bms, res["ms_per_step"], sm["gemm_flops"])
            entry["mfu_accounting"] = mfu_accounting(sm["value"], entry["bf16_comparison"]["tflops"], peaks)
        del res["step"]
        torch.cuda.empty_cache()
        if not args.no_e2e:
            e = run_e2e(wl, dev, K=min(K, e2e_steps(wl)), warmup=1, accum=A)
            entry["e2e"] = {"value": round(sm["gemm_flops"] / (e["ms_per_step"] * 1e-3) / 1e12, 2),
                            "unit": "TFLOP/s", "ms_per_step": round(e["ms_per_step"], 3),
                            "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"]}
        torch.cuda.empty_cache()
        if not args.no_cpu_baseline:
            entry["cpu_baseline"] = cpu_baseline(wl, min_s=2.0)
        out[workload_tag(name, m)] = entry
        del wl
    return out


def bf16_step_ms(step, K):
    """The same linear step in BF16 through cuBLAS (torch.matmul): per layer
    Y = X W^T, dX = dY W, dW = dY^T X, on the same device input sets, K steps
    captured in one CUDA graph and timed with device events.  This is the
    FP8-vs-BF16 comparison of the pages' throughput claim, taken at the level
    of the linear layers."""
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
    del g, outs
    return ms


def mfu_accounting(fp8_tflops, bf16_tflops, peaks):
    """Mixed-precision MFU bookkeeping with the pages' weighting: 72 % of a
    step's FLOPs in FP8 linear layers, 28 % in BF16.  The effective peak is the
    time-weighted (harmonic) mean P_eff = (0.72/P_fp8 + 0.28/P_bf16)^-1; the
    projected throughput combines the measured FP8 linear-layer rate with the
    measured BF16 cuBLAS rate on the same shapes for the BF16 share."""
    f8, bf = 0.72, 0.28
    nominal = {"fp8": SPEC_FP8_TFLOPS, "bf16": SPEC_BF16_TFLOPS}
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
    torch's scaled_mm, at 8192^3 and at the GEMM shapes of the step.  Not the
    same scaling granularity as the path (1x128 / 128x128), so it is a
    ceiling estimate, not a comparison arm.  None if unavailable."""
    import torch
    import torch.nn.functional as F
    if not hasattr(F, "scaled_mm") or not hasattr(torch, "float8_e8m0fnu"):
        return None

    def rup(a, b):
        return (a + b - 1) // b * b

    def timed(m, n, k, reps=10):
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
        del a, b, sa, sb
        return ms

    try:
        ms = timed(8192, 8192, 8192)
        peak = 2.0 * 8192 ** 3 / (ms * 1e-3) / 1e12
        tot_ms, tot_flops = 0.0, 0
        for L in wl.layers:
            for (m, n, k) in ((L.m, L.n, L.k), (L.m, L.k, L.n), (L.n, L.k, L.m)):
                tot_ms += timed(m, n, k)
                tot_flops += 2 * m * n * k
        torch.cuda.empty_cache()
        return {"source": "cuBLASLt MXFP8 via torch scaled_mm (1x32 UE8M0 scales, BF16 out)",
                "tflops_8192cube": round(peak, 1),
                "tflops_step_shapes": round(tot_flops / (tot_ms * 1e-3) / 1e12, 1)}
    except Exception as e:  # noqa: BLE001  (library path missing on this build)
        return {"unavailable": str(e).splitlines()[0][:160]}


def gemm_sustained(step, dev, gpu, seconds=1.0, rounds=2):
    """Our GEMM launches against cuBLASLt's MXFP8 GEMM in the same regime: the
    step's GEMMs alone (fprop and the fused dgrad + wgrad of every layer),
    and the library's GEMM on the SAME E4M3 codes and shapes (fprop, dgrad,
    wgrad per layer; the library takes 1x32 UE8M0 scales, all set to 1.0,
    and writes BF16 where our wgrad adds FP32 into the main grads).  Each
    side is one CUDA graph of a step's GEMMs replayed back to back for about
    `seconds`, so both run as long, power-capped loops; the sides alternate
    `rounds` times and the clocks are sampled over each.  None if the
    library path is missing."""
    import torch
    import torch.nn.functional as F
    if not hasattr(F, "scaled_mm") or not hasattr(torch, "float8_e8m0fnu"):
        return None
    fp8 = step.fp8
    e4m3 = torch.float8_e4m3fn

    def rup(a, b):
        return (a + b - 1) // b * b

    ones = {}

    def unit_scales(rows, k):
        key = (rows, k)
        if key not in ones:
            ones[key] = torch.full((rup(rows, 128) * rup(k // 32, 4),), 127, dtype=torch.uint8,
                                   device=dev).view(torch.float8_e8m0fnu)
        return ones[key]

    lib_ops, flops = [], 0
    for L, (xq, wq, dyq, _y, _dx) in zip(step.layers, step.out):
        m, n, k = L.m, L.n, L.k
        ops = ((xq.q, wq.q, m, n, k),                       # Y  = X W^T
               (dyq.q, wq.qt, m, k, n),                     # dX = dY W
               (dyq.qt[:, :m], xq.qt[:, :m], n, k, m))      # dW = dY^T X
        for a, b, rows, cols, kk in ops:
            lib_ops.append((a.view(e4m3), b.view(e4m3), unit_scales(rows, kk), unit_scales(cols, kk)))
            flops += 2 * rows * cols * kk

    def ours():
        for li, (xq, wq, dyq, y, dx) in enumerate(step.out):
            fp8.gemm_fprop(xq, wq, out=y)
            fp8.gemm_dgrad_wgrad(dyq, wq, xq, dx=dx, dw=step.grads[li], accumulate=True)

    def library():
        for a, b, sa, sb in lib_ops:
            F.scaled_mm(a, b.t(), sa, F.ScalingType.BlockWise1x32, sb, F.ScalingType.BlockWise1x32,
                        swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                        output_dtype=torch.bfloat16)

    try:
        graphs = {}
        cap = torch.cuda.Stream()
        cap.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(cap):
            for name, fn in (("ours", ours), ("library", library)):
                fn()  # outside the graph first: library workspaces, attribute setup
                torch.cuda.synchronize()
                graphs[name] = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graphs[name], stream=cap):
                    fn()
        torch.cuda.synchronize()
        res = {name: [] for name in graphs}
        for _ in range(rounds):
            for name, g in graphs.items():
                g.replay()
                t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                t0.record(); g.replay(); t1.record()
                torch.cuda.synchronize()
                reps = max(3, int(seconds * 1e3 / max(t0.elapsed_time(t1), 1e-3)))
                with ClockSampler(gpu) as clk:
                    t0.record()
                    for _ in range(reps):
                        g.replay()
                    t1.record()
                    torch.cuda.synchronize()
                ms = t0.elapsed_time(t1) / reps
                res[name].append({"tflops": round(flops / (ms * 1e-3) / 1e12, 1),
                                  "sm_mhz": clk.summary().get("sm_mhz"), "reps": reps})
        if fp8.device_status() != 0:
            raise RuntimeError("device status %d" % fp8.device_status())
        del graphs
        torch.cuda.empty_cache()
    except Exception as e:  # noqa: BLE001  (library path missing on this build)
        return {"unavailable": str(e).splitlines()[0][:160]}
    mean = {name: round(statistics.mean(r["tflops"] for r in v), 1) for name, v in res.items()}
    return {"what": "the step's GEMMs alone, ours vs cuBLASLt MXFP8 on the same E4M3 codes and "
                    "shapes, each a graph replayed back to back for ~%.1f s, alternating %d times"
                    % (seconds, rounds),
            "gemm_flops_per_pass": flops,
            "ours_tflops": mean["ours"], "library_tflops": mean["library"],
            "ours_vs_library": round(mean["ours"] / mean["library"], 3),
            "rounds": res}


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
    if fp8.device_status() != 0:
        raise RuntimeError("device status after the end-to-end run")
    windows = (K + accum - 1) // accum
    out = {"ms_per_step": s.elapsed_time(e) / K, "steps": K,
           "h2d": int(bytes_in + bytes_w * windows / K),
           "d2h": int(bytes_out + bytes_dw * windows / K)}
    del host_w, host_in, host_out, host_dw, dev_w, dev_in, results, grads, wq
    return out


# ---------------------------------------------------------------- CPU oracle

def oracle_threads() -> int:
    """Gives the oracle's OpenMP loops every core this process may run on
    (torchrun sets OMP_NUM_THREADS=1 for its ranks) and returns the number of
    threads its parallel regions will use."""
    import ctypes
    import oracle
    oracle._load()
    n = len(os.sched_getaffinity(0))
    try:
        gomp = ctypes.CDLL("libgomp.so.1")
    except OSError:
        return 1 if os.environ.get("OMP_NUM_THREADS") == "1" else n
    gomp.omp_set_num_threads(n)
    return int(gomp.omp_get_max_threads())


def _sample_idx(total, r):
    import numpy as np
    return np.unique(np.linspace(0, total - 1, min(r, total)).astype(np.int64))


def _oracle_sample(wl, r):
    """The hot path on a bounded sample, through the CPU oracle: for every
    layer, r output rows of fprop and of dgrad and an r x r block of wgrad's
    output, each with the quantization those outputs need (the rows of X or dY
    and the whole weight for fprop/dgrad; the r columns of dY and of X, over
    all tokens, for wgrad).  Returns the sampled GEMM FLOPs."""
    import oracle

    flops = 0
    for L in wl.layers:
        m, n, k = L.m, L.n, L.k
        rows = _sample_idx(m, r)
        oracle.linear_fprop(L.x[rows], L.w)
        oracle.linear_dgrad(L.dy[rows], L.w)
        ncols, kcols = _sample_idx(n, r), _sample_idx(k, r)
        oracle.linear_wgrad(L.dy[:, ncols].contiguous(), L.x[:, kcols].contiguous())
        flops += 2 * 2 * rows.size * n * k + 2 * ncols.size * kcols.size * m
    return flops


def cpu_baseline(wl, min_s=10.0):
    """Times the oracle on a sample of the workload that takes at least `min_s`
    seconds: the sample size doubles until one sample run lasts that long (the
    last run is the reported one, so it lasts between `min_s` and about twice
    that)."""
    n_cores = oracle_threads()
    r = 16
    while True:
        t0 = time.perf_counter()
        f = _oracle_sample(wl, r)
        dt = time.perf_counter() - t0
        if dt >= min_s or r >= 8192:
            break
        r *= 2
    return {"value": round(f / dt / 1e12, 6), "unit": "TFLOP/s", "cores": n_cores,
            "kind": "oracle",
            "sample": "%d output rows of each fprop and dgrad and a %dx%d block of each wgrad "
                      "(all layers) with the quantization they need, FP64 C oracle, %.1f s"
                      % (r, r, r, dt)}


def run_reference(args):
    """Reference arm: the CPU oracle as it stands, on a bounded sample of the
    same workload per step; rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl = make_workload(args.workload, args.m)
    n_cores = oracle_threads()
    r = 8
    for _ in range(args.warmup):
        _oracle_sample(wl, r)
    t0 = time.perf_counter()
    flops = 0
    for _ in range(args.steps):
        flops += _oracle_sample(wl, r)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = ("%d output rows of each fprop and dgrad and a %dx%d block of each wgrad per step "
              "(all layers) with the quantization they need, FP64 C oracle" % (r, r, r))
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3 / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": workload_tag(args.workload, args.m),
                   "layers": WORKLOADS[args.workload][2], "tokens_per_gpu": args.m,
                   "seed": WORKLOADS[args.workload][1]},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": n_cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- launch

def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def spawn_ranks(args, argv):
    """--gpus N > 1 outside torchrun: start N ranks with torch.distributed.run
    on this node, relay their output, and fail unless exactly one JSON line
    for N GPUs came out."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", str(args.gpus), "--master-addr", "127.0.0.1",
           "--master-port", str(_free_port()), os.path.abspath(__file__)] + list(argv)
    env = dict(os.environ)
    if args.impl == "ours":
        env.setdefault("NCCL_DEBUG", "INFO")
    proc = subprocess.run(cmd, env=env, stdout=subprocess.PIPE, text=True, timeout=3600)
    lines = [l for l in proc.stdout.splitlines() if l.startswith("{")]
    for l in proc.stdout.splitlines():
        print(l, flush=True)
    if proc.returncode != 0:
        return proc.returncode
    if len(lines) != 1 or json.loads(lines[0]).get("n_gpus") != args.gpus:
        print("bench.py: expected one JSON line for %d GPUs from the ranks" % args.gpus, file=sys.stderr)
        return 1
    return 0


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    args = _parse_args(argv)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args, argv))
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
