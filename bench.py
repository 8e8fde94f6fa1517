#!/usr/bin/env python
"""Throughput of the B200 FP8 W8A8 linear layer on one workload.

A step is one forward pass of the workload's FP8 linears: every distinct
activation is quantized (dynamic per-token or per-128-group scales), then
every GEMM runs.  Weights are quantized once at load time, outside the step
(that kernel is timed separately and reported under "weight_quant").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle, timed on a sample

The L2 cache (126 MB) is flushed before every step and before every timed
op: a 256 MiB buffer is written, then another 256 MiB buffer is read, so the
timed kernels start with a cold L2 that holds no dirty lines (a write alone
would leave 126 MB of dirty lines for the timed kernel to write back).  Each
step and each kernel launch is timed with CUDA events on the launching stream,
so the flush is not counted.  With N > 1 (torchrun, one rank per GPU) every
rank runs its own batch of tokens against replicated weights (token-parallel,
no collective on the data path): weak scaling, value = all ranks' work over
the slowest rank's time.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

DEFAULT_WORKLOAD = "llama3.1-70b_sweep"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_OVER_BF16 = 2.0        # nominal dense fp8 / bf16 tensor ratio (4.5 / 2.25 PFLOP/s)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fp8q", choices=["fp8q", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--flush-mib", type=int, default=256)
    ap.add_argument("--cpu-sample-rows", type=int, default=16,
                    help="rows of every GEMM the CPU oracle starts its cpu_baseline sample with")
    ap.add_argument("--ref-sample-rows", type=int, default=8,
                    help="rows of every GEMM one reference-arm step runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch every op from Python each step instead of replaying CUDA graphs")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the next-step sections (RMSNorm, SwiGLU, static scales, KV cache, weight-only, "
                         "merged GEMMs): for short profiling runs")
    ap.add_argument("--only", default="",
                    help="comma-separated GEMM names: restrict the workload to them (profiling)")
    return ap.parse_args()


def select(args):
    wl = synth.workloads()[args.workload]
    if args.only:
        keep = set(args.only.split(","))
        wl = synth.Workload(wl.name + "[" + args.only + "]", [g for g in wl.gemms if g.name in keep])
        if not wl.gemms:
            raise SystemExit(f"--only {args.only}: no such GEMM in {args.workload}")
    return wl


def peaks():
    try:
        p = json.load(open(PEAKS_FILE))
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def metric_for(wl) -> tuple:
    decode = all(g.M <= 16 for g in wl.gemms)
    if decode:
        return "FP8 linear GB/s vs HBM (decode M<=16)", "GB/s"
    return "FP8 linear TFLOP/s and % of FP8 peak (prefill)", "TFLOP/s"


def gemm_bytes(g) -> int:
    """Algorithmic bytes of one FP8 linear: codes of X and W once, bf16 Y
    once, and the scales."""
    if g.mode == synth.CHANNEL_TOKEN:
        sb = 4 * g.M + 4 * g.N
    else:
        sb = 4 * g.M * (g.K // 128) + 4 * ((g.N + 127) // 128) * (g.K // 128)
    return g.M * g.K + g.N * g.K + 2 * g.M * g.N + sb


def quant_bytes(rows, K, mode) -> int:
    nscale = rows if mode == synth.CHANNEL_TOKEN else rows * (K // 128)
    return 2 * rows * K + rows * K + 4 * nscale


def step_units(wl, unit) -> float:
    """Work of one step in the metric's unit numerator (flop or byte)."""
    if unit == "GB/s":
        xs = {}
        for g in wl.gemms:
            xs[g.x] = (g.M, g.K, g.mode)
        return float(sum(gemm_bytes(g) for g in wl.gemms) + sum(quant_bytes(*v) for v in xs.values()))
    return float(sum(g.flops for g in wl.gemms))


def to_metric(units, seconds, unit):
    return units / seconds / (1e9 if unit == "GB/s" else 1e12)


# ------------------------------------------------------------------ clocks ---

_CLOCK_WORKER = r"""
import json, select, sys, time
reasons = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}
index, period = int(sys.argv[1]), float(sys.argv[2])
try:
    import pynvml
    pynvml.nvmlInit()
    h = pynvml.nvmlDeviceGetHandleByIndex(index)
    mx = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
except Exception as e:
    print(json.dumps({"error": "nvml unavailable: %s" % e}), flush=True)
    sys.exit(0)
print(json.dumps({"ready": True}), flush=True)
samples, seen = [], set()
while True:
    r, _, _ = select.select([sys.stdin], [], [], period)
    if r:
        break
    try:
        samples.append(pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM))
        ev = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
        seen.update(name for bit, name in reasons.items() if ev & bit)
    except Exception as e:
        print(json.dumps({"error": str(e)}), flush=True)
        sys.exit(0)
print(json.dumps({"samples": samples, "reasons": sorted(seen), "max": mx}), flush=True)
"""


class ClockSampler:
    """NVML samples of the SM clock and clock-event reasons, taken by a
    separate small process (no GIL shared with the launching thread) for as
    long as the timed region runs."""

    def __init__(self, index: int, period_s: float = 0.001):
        self.index, self.period = index, period_s
        self.result = {"error": "not run"}

    def __enter__(self):
        self.proc = subprocess.Popen([sys.executable, "-c", _CLOCK_WORKER, str(self.index), str(self.period)],
                                     stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True)
        first = json.loads(self.proc.stdout.readline() or '{"error": "sampler exited"}')
        self.ok = "ready" in first
        if not self.ok:
            self.result = first
        return self

    def __exit__(self, *a):
        try:
            out, _ = self.proc.communicate(input="stop\n", timeout=60)
            if self.ok:
                self.result = json.loads(out.strip().splitlines()[-1])
        except Exception as e:
            self.proc.kill()
            self.result = {"error": f"sampler: {e}"}

    def summary(self):
        r = self.result
        if "samples" not in r or not r["samples"]:
            return {"sm_mhz": None, "sm_max_mhz": r.get("max"), "reasons": r.get("reasons", []),
                    "samples": 0, "error": r.get("error")}
        smp = r["samples"]
        return {"sm_mhz": float(statistics.median(smp)), "sm_max_mhz": r["max"], "sm_mhz_min": float(min(smp)),
                "reasons": [x for x in r["reasons"] if x != "gpu_idle"], "samples": len(smp),
                "sampler": "NVML in a separate process, every 1 ms during the timed steps"}


_MONITOR_SRC = r"""
extern "C" __global__ void clock_monitor(unsigned long long duration_ns, unsigned long long* out, int max_samples) {
  // One thread: every ~0.5 ms record (clock64, globaltimer) of this SM, for
  // duration_ns of wall time or max_samples samples, whichever comes first.
  unsigned long long t0, t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
  for (int i = 0; i < max_samples; ++i) {
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    out[2 * i] = clock64();
    out[2 * i + 1] = t;
    if (t - t0 > duration_ns) { out[2 * i + 2] = 0; return; }
    for (int k = 0; k < 10; ++k) __nanosleep(50000);
  }
}
"""


class ClockMonitor:
    """Measures the SM clock the kernels actually run at: a one-warp kernel
    on a side stream records this SM's cycle counter against the global
    nanosecond timer while the timed steps run (NVML's reading lags by tens
    of milliseconds and misses power capping in short runs)."""

    def __init__(self, duration_s: float, max_samples: int = 4096):
        self.err, self.samples = None, None
        try:
            import tempfile
            from cuda.bindings import driver as cu
            self.cu = cu
            d = tempfile.mkdtemp(prefix="clkmon")
            src, cub = os.path.join(d, "m.cu"), os.path.join(d, "m.cubin")
            open(src, "w").write(_MONITOR_SRC)
            nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
            subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-cubin", "-o", cub, src],
                                  stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            err, self.mod = cu.cuModuleLoad(cub.encode())
            err2, self.fn = cu.cuModuleGetFunction(self.mod, b"clock_monitor")
            if int(err) or int(err2):
                raise RuntimeError(f"module load: {err} {err2}")
            self.max = max_samples
            self.buf = torch.zeros(2 * max_samples + 2, dtype=torch.int64, device="cuda")
            self.duration_ns = int(duration_s * 1e9)
            self.stream = torch.cuda.Stream()
        except Exception as e:
            self.err = f"clock monitor unavailable: {e}"

    def start(self):
        if self.err:
            return
        import ctypes
        self._args = (ctypes.c_ulonglong(self.duration_ns), ctypes.c_void_p(self.buf.data_ptr()),
                      ctypes.c_int(self.max))
        self._ptrs = (ctypes.c_void_p * 3)(*[ctypes.addressof(a) for a in self._args])
        (r,) = self.cu.cuLaunchKernel(self.fn, 1, 1, 1, 1, 1, 1, 0, self.stream.cuda_stream,
                                      ctypes.addressof(self._ptrs), 0)
        if int(r):
            self.err = f"clock monitor launch: {r}"

    def summary(self):
        if self.err:
            return {"error": self.err}
        torch.cuda.synchronize()
        v = self.buf.cpu().numpy().reshape(-1, 2)
        v = v[: np.argmax(v[:, 1] == 0)] if np.any(v[:, 1] == 0) else v
        if len(v) < 3:
            return {"error": "too few samples"}
        mhz = np.diff(v[:, 0]) / np.diff(v[:, 1]) * 1e3
        return {"sm_mhz_median": round(float(np.median(mhz)), 1), "sm_mhz_min": round(float(mhz.min()), 1),
                "intervals": int(mhz.size),
                "method": "clock64 / %globaltimer on one SM, ~0.5 ms intervals, during an untimed repeat of the steps"}


# --------------------------------------------------------------- GPU arm ---

def dist_setup(args, backend="nccl"):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _collective_device():
    return "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"


def max_over_ranks(v, world):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=_collective_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(v, world):
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=_collective_device())
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def x_seed(rank: int, i: int) -> int:
    """Seed of the i-th activation of rank `rank`: every rank quantizes and
    multiplies its own batch of tokens (token-parallel, weights replicated)."""
    return 1000 * rank + i


def aggregate(units_local: float, seconds_local: float, world: int):
    """Whole-job work over the slowest rank's time (weak scaling)."""
    return sum_over_ranks(units_local, world), max_over_ranks(seconds_local, world)


def decode_reduce_launched(g, sms: int) -> bool:
    """Whether fp8_linear launches its separate split-sum kernel after the
    decode GEMM (M <= 64): the library's dispatch rule, restated for counting."""
    if g.M > 64:
        return False
    n_tiles, kb = -(-g.N // 128), -(-g.K // 128)
    total = n_tiles * kb
    G = min(total, sms)
    nx = 16 if g.M <= 16 else (32 if g.M <= 32 else 64)
    if g.mode == synth.BLOCK128:
        # cluster split-K (no second kernel) where clusters of C in [2, 8] CTAs,
        # one weight tile each, fill at least 3/4 of the SMs (assuming the
        # device holds that many clusters at once, as the library checks)
        C = min(8, sms // n_tiles, kb)
        return not (C >= 2 and 4 * n_tiles * C >= 3 * sms)
    return not (nx == 16 or total >= kb * G)


def launches_of(g, sms: int) -> int:
    return 1 + int(decode_reduce_launched(g, sms))


def graph_kernel_nodes(graph):
    """Kernel launches in a captured CUDA graph (its kernel nodes), or None
    where the graph cannot be inspected."""
    try:
        from cuda.bindings import runtime as rt
        h = rt.cudaGraph_t(init_value=graph.raw_cuda_graph())
        err, _, n = rt.cudaGraphGetNodes(h, 0)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        err, nodes, n = rt.cudaGraphGetNodes(h, n)
        if err != rt.cudaError_t.cudaSuccess:
            return None
        count = 0
        for node in nodes[:n]:
            err, kind = rt.cudaGraphNodeGetType(node)
            if err != rt.cudaError_t.cudaSuccess:
                return None
            count += int(kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel)
        return count
    except Exception:
        return None


def config_of(wl, world: int, flush_mib: int) -> dict:
    """The workload description both arms print (the same dict for the same run)."""
    return {"workload": wl.name,
            "gemms": [f"{g.name}:{g.M}x{g.K}->{g.N}:{'channel' if g.mode == 0 else 'block128'}" for g in wl.gemms],
            "weights": sorted({g.weight for g in wl.gemms}),
            "step": "quantize each activation + every FP8 GEMM; weights quantized at load",
            "l2": f"GPU arm: L2 flushed before every step and every timed op, outside the timed events: a "
                  f"{flush_mib} MiB buffer written, then another {flush_mib} MiB read (cold, clean L2)",
            "parallelism": "single device" if world == 1 else f"token-parallel x{world}, weights replicated"}


def run_gpu(args):
    world, rank, local = dist_setup(args)
    torch.cuda.set_device(local)
    import fp8_w8a8_quantized_amax_b200 as fq
    from fp8_w8a8_quantized_amax_b200 import build as fbuild
    fbuild.build()
    dev = torch.device("cuda", local)
    wl = select(args)
    metric, unit = metric_for(wl)
    pk = peaks()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    # ---- load time: weights (replicated), quantized once
    W = {}
    for g in wl.gemms:
        if g.weight in W:
            continue
        seed = synth.weight_seed(g.weight)
        W[g.weight] = synth.make_w(g.N, g.K, seed=seed).to(dev) if g.N * g.K <= (1 << 26) \
            else synth.make_w_device(g.N, g.K, seed=seed, device=dev)
    xs_shapes = {}
    for g in wl.gemms:
        xs_shapes.setdefault(g.x, (g.M, g.K, g.mode))
    X = {k: synth.make_x_device(M, K, seed=x_seed(rank, i), device=dev)
         for i, (k, (M, K, _)) in enumerate(xs_shapes.items())}
    WQ = {}
    for g in wl.gemms:
        if g.weight not in WQ:
            WQ[g.weight] = fq.fp8_quant_weight(W[g.weight], g.mode)
    XQ = {k: (torch.empty((M, K), dtype=torch.uint8, device=dev),
              torch.empty(fq.scale_shape_act(M, K, mode), dtype=torch.float32, device=dev))
          for k, (M, K, mode) in xs_shapes.items()}
    Y = {g.name: torch.empty((g.M, g.N), dtype=torch.bfloat16, device=dev) for g in wl.gemms}
    # scratch of the decode path and of the stream-K prefill schedule (where
    # fp8_linear_workspace_size asks for one), zero-filled once
    WS = {}
    for g in wl.gemms:
        nws = fq.fp8_linear_workspace_size(g.M, g.N, g.K, g.mode)
        WS[g.name] = torch.zeros(nws, dtype=torch.uint8, device=dev) if nws else None
    class _Flush:
        """Write one buffer larger than L2, then read another: L2 ends up
        holding only clean lines of the read buffer."""

        def __init__(self, mib):
            self.w = torch.empty(mib << 20, dtype=torch.uint8, device=dev)
            self.r = torch.ones(mib << 17, dtype=torch.int64, device=dev)
            self.sink = torch.empty((), dtype=torch.int64, device=dev)

        def zero_(self):
            self.w.zero_()
            torch.amax(self.r, dim=0, out=self.sink)

    flush = _Flush(args.flush_mib)
    stream = torch.cuda.current_stream(dev)

    n_ops = len(xs_shapes) + len(wl.gemms)

    def make_ops():
        ops = []
        for k, (M, K, mode) in xs_shapes.items():
            ops.append(lambda k=k, mode=mode: fq.fp8_quant_act(X[k], mode, out=XQ[k]))
        for g in wl.gemms:
            def op(g=g):
                xq, xsc = XQ[g.x]
                wq, wsc = WQ[g.weight]
                fq.fp8_linear(xq, xsc, wq, wsc, g.mode, out=Y[g.name], workspace=WS[g.name])
            ops.append(op)
        return ops

    ops = make_ops()
    for _ in range(args.warmup):
        flush.zero_()
        for op in ops:
            op()
    torch.cuda.synchronize()
    assert fq.device_error(clear=True) == 0

    def capture(fns, keep=False):
        g = torch.cuda.CUDAGraph(keep_graph=keep)
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for f in fns:
                    f()
        stream.wait_stream(side)
        torch.cuda.synchronize()
        return g

    # The step as one CUDA graph (kernels of consecutive ops overlap their
    # launch through programmatic dependent launch); each op also as its own
    # graph, timed alone for the per-kernel figures.
    launches_per_step = len(xs_shapes) + sum(launches_of(g, sms) for g in wl.gemms)
    launches_source = "the library's dispatch rule, restated (decode_reduce_launched)"
    if args.eager:
        step_runner = lambda: [op() for op in ops]
        op_runners = ops
    else:
        step_graph = capture(ops, keep=True)    # kept, to count its kernel nodes
        counted = graph_kernel_nodes(step_graph)
        if counted is not None:
            launches_per_step, launches_source = counted, "kernel nodes of the captured step graph"
        step_graph.instantiate()
        op_graphs = [capture([op]) for op in ops]
        step_runner = step_graph.replay
        op_runners = [g.replay for g in op_graphs]
        for _ in range(2):
            step_runner()
            for r in op_runners:
                r()
        torch.cuda.synchronize()

    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    # expected length of the timed loop, for the clock monitor
    t_est = time.perf_counter()
    for _ in range(3):
        flush.zero_()
        step_runner()
    torch.cuda.synchronize()
    loop_s = (time.perf_counter() - t_est) / 3 * args.steps
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        torch.cuda._sleep(2_000_000)          # lets the host queue ahead of the device
        for s in range(args.steps):
            flush.zero_()
            step_ev[s][0].record(stream)
            step_runner()
            step_ev[s][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    # The clock the kernels actually ran at, measured on an untimed repeat of
    # the same steps (the monitor's warp occupies one SM, so it stays out of
    # the timed loop).
    mon = ClockMonitor(duration_s=loop_s + 0.005)
    mon.start()
    for _ in range(args.steps):
        flush.zero_()
        step_runner()
    torch.cuda.synchronize()
    units = step_units(wl, unit) * args.steps
    all_units, total_s = aggregate(units, sum(step_ms) / 1e3, world)
    value = to_metric(all_units, total_s, unit)

    # per-op times.  (1) isolated: each op's own graph, one launch after its
    # own L2 flush -- the launch latency of a lone kernel included.  (2)
    # back to back: R launches of the op in one graph, over R sets of buffers
    # (copies of its inputs and outputs) whose footprint together is at least
    # twice L2, so that every launch reads its inputs from DRAM; per launch =
    # the graph's time / R, after an L2 flush.  (2) is what "ms" reports.
    op_ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_ops)] for _ in range(args.steps)]
    torch.cuda._sleep(2_000_000)
    for s in range(args.steps):
        for i, r in enumerate(op_runners):
            flush.zero_()
            op_ev[s][i][0].record(stream)
            r()
            op_ev[s][i][1].record(stream)
    torch.cuda.synchronize()
    op_ms_isolated = np.array([[a.elapsed_time(b) for a, b in row] for row in op_ev]).mean(axis=0)
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    xs_items = list(xs_shapes.items())

    def rotating(i):
        """(R, functions): R launches of op i over R buffer sets."""
        if i < len(xs_items):
            k, (M, K, mode) = xs_items[i]
            R = int(min(32, max(2, -(-2 * l2_bytes // quant_bytes(M, K, mode)))))
            xs_ = [X[k]] + [X[k].clone() for _ in range(R - 1)]
            outs = [XQ[k]] + [(torch.empty_like(XQ[k][0]), torch.empty_like(XQ[k][1])) for _ in range(R - 1)]
            return R, [lambda x=x, o=o, mode=mode: fq.fp8_quant_act(x, mode, out=o) for x, o in zip(xs_, outs)]
        g = wl.gemms[i - len(xs_items)]
        R = int(min(32, max(2, -(-2 * l2_bytes // gemm_bytes(g)))))
        xq, xsc = XQ[g.x]
        wq, wsc = WQ[g.weight]
        sets = [(xq, xsc, wq, wsc, Y[g.name], WS[g.name])]
        for _ in range(R - 1):
            sets.append((xq.clone(), xsc.clone(), wq.clone(), wsc.clone(), torch.empty_like(Y[g.name]),
                         torch.zeros_like(WS[g.name]) if WS[g.name] is not None else None))
        return R, [lambda st=st, g=g: fq.fp8_linear(st[0], st[1], st[2], st[3], g.mode, out=st[4], workspace=st[5])
                   for st in sets]

    LONG_OP_MS = 0.25
    op_ms = np.zeros(n_ops)
    op_reps = [1] * n_ops
    for i in range(n_ops):
        R, fns = rotating(i)
        for f in fns:
            f()
        torch.cuda.synchronize()
        gr = capture(fns) if not args.eager else None
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda._sleep(1_000_000)
        for s_ in range(args.steps):
            flush.zero_()
            ev[s_][0].record(stream)
            if gr is not None:
                gr.replay()
            else:
                for f in fns:
                    f()
            ev[s_][1].record(stream)
        torch.cuda.synchronize()
        op_ms[i] = float(np.mean([a.elapsed_time(b) for a, b in ev])) / R
        op_reps[i] = R
        del gr, fns
        if op_ms_isolated[i] >= LONG_OP_MS:
            # a long kernel is reported as timed alone: its launch latency is a
            # few percent of it, and two back to back already run into the
            # power cap (its roofline uses the burst peak, measured alone)
            op_ms[i] = op_ms_isolated[i]
            op_reps[i] = 1
    torch.cuda.empty_cache()
    err = fq.device_error(clear=True)

    # ---- GEMMs that read the same activation, run as one GEMM over their
    # stacked weights (what serving engines do with q/k/v or gate/up); the
    # per-channel and 128x128-block scales are row-local, so stacking the
    # quantized weights and scales is exact.
    merged = None
    groups = {}
    for g in wl.gemms:
        groups.setdefault((g.x, g.mode), []).append(g)
    if not args.eager and not args.no_extras and any(len(v) > 1 for v in groups.values()):
        mops, mnames = [], []
        for (xk, mode), gs in groups.items():
            if len(gs) == 1:
                g = gs[0]
                mops.append(lambda g=g: fq.fp8_linear(XQ[g.x][0], XQ[g.x][1], WQ[g.weight][0], WQ[g.weight][1], g.mode,
                                                      out=Y[g.name], workspace=WS[g.name]))
                mnames.append(g.name)
                continue
            wq_m = torch.cat([WQ[g.weight][0] for g in gs])
            ws_m = torch.cat([WQ[g.weight][1] for g in gs])
            M, K, Nm = gs[0].M, gs[0].K, sum(g.N for g in gs)
            y_m = torch.empty((M, Nm), dtype=torch.bfloat16, device=dev)
            nws = fq.fp8_linear_workspace_size(M, Nm, K, mode)
            ws_buf = torch.zeros(nws, dtype=torch.uint8, device=dev) if nws else None
            mops.append(lambda xk=xk, mode=mode, wq_m=wq_m, ws_m=ws_m, y_m=y_m, ws_buf=ws_buf:
                        fq.fp8_linear(XQ[xk][0], XQ[xk][1], wq_m, ws_m, mode, out=y_m, workspace=ws_buf))
            mnames.append("+".join(g.name for g in gs) + f":{M}x{K}->{Nm}")
        qops = ops[:len(xs_shapes)]
        for f in qops + mops:
            f()
        torch.cuda.synchronize()
        mgraph = capture(qops + mops)
        for _ in range(2):
            mgraph.replay()
        mev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda._sleep(2_000_000)
        for s_ in range(args.steps):
            flush.zero_()
            mev[s_][0].record(stream)
            mgraph.replay()
            mev[s_][1].record(stream)
        torch.cuda.synchronize()
        mt = sum(a.elapsed_time(b) for a, b in mev) / 1e3
        merged = {"value": round(to_metric(units, mt, unit), 3), "unit": unit,
                  "ms_per_step": round(mt * 1e3 / args.steps, 4), "gemms": mnames,
                  "note": "same step, GEMMs sharing an input launched as one GEMM over stacked weights"}

    # ---- per-kernel detail and the rooflines: the dominant kernel of the
    # step, and the dominant prefill GEMM, decode GEMM and quantize launch
    names = [f"quant_act[{k}]" for k in xs_shapes] + [g.name for g in wl.gemms]
    detail = []
    fp8_peak = pk["bf16_tflops"] * FP8_OVER_BF16
    for i, (k, (M, K, mode)) in enumerate(xs_shapes.items()):
        b = quant_bytes(M, K, mode)
        detail.append({"op": names[i], "kernel": "quant_rows" if mode == 0 else "quant_groups128", "bound": "hbm",
                       "M": M, "K": K, "mode": mode, "back_to_back": op_reps[i],
                       "ms_isolated": round(float(op_ms_isolated[i]), 5),
                       "ms": round(float(op_ms[i]), 5), "GB/s": round(b / (op_ms[i] / 1e3) / 1e9, 1),
                       "frac_hbm": round(b / (op_ms[i] / 1e3) / 1e9 / pk["hbm_gbs"], 3)})
    for j, g in enumerate(wl.gemms):
        t = op_ms[len(xs_shapes) + j] / 1e3
        kern = ("gemm_decode" if g.M <= 64 else
                ("gemm_block" if g.mode == synth.BLOCK128 else "gemm_channel"))
        detail.append({"op": g.name, "kernel": kern, "bound": "hbm" if g.M <= 64 else "tensor",
                       "M": g.M, "N": g.N, "K": g.K, "mode": g.mode, "back_to_back": op_reps[len(xs_shapes) + j],
                       "ms_isolated": round(float(op_ms_isolated[len(xs_shapes) + j]), 5),
                       "ms": round(float(op_ms[len(xs_shapes) + j]), 5),
                       "TFLOP/s": round(g.flops / t / 1e12, 1),
                       "GB/s": round(gemm_bytes(g) / t / 1e9, 1),
                       "frac_fp8_peak": round(g.flops / t / 1e12 / fp8_peak, 3),
                       "frac_hbm": round(gemm_bytes(g) / t / 1e9 / pk["hbm_gbs"], 3)})
    gemm_by_name = {g.name: g for g in wl.gemms}
    traffic = {}
    tfile = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tfile):
        try:
            traffic = json.load(open(tfile))
        except Exception:
            traffic = {}

    def roofline_of(d):
        if d["bound"] == "tensor":
            g = gemm_by_name[d["op"]]
            r = {"op": d["op"], "kernel": d["kernel"], "bound": "tensor", "achieved": d["TFLOP/s"],
                 "peak": round(fp8_peak, 1), "unit": "TFLOP/s", "frac": round(d["TFLOP/s"] / fp8_peak, 3),
                 "peak_basis": f"{pk['source']} bf16 burst {pk['bf16_tflops']} TFLOP/s x {FP8_OVER_BF16} "
                               "(nominal fp8/bf16 dense ratio), of measured",
                 "algorithmic": f"2*M*N*K = {g.flops} flop per launch", "traffic": None}
        else:
            if d["op"] in gemm_by_name:
                alg = f"M*K + N*K + 2*M*N + scales = {gemm_bytes(gemm_by_name[d['op']])} bytes per launch"
            else:
                alg = f"2*M*K (bf16 in) + M*K (codes) + 4 per scale = {quant_bytes(d['M'], d['K'], d['mode'])} bytes per launch"
            r = {"op": d["op"], "kernel": d["kernel"], "bound": "hbm", "achieved": d["GB/s"], "peak": pk["hbm_gbs"],
                 "unit": "GB/s", "frac": round(d["GB/s"] / pk["hbm_gbs"], 3),
                 "peak_basis": f"{pk['source']} HBM copy bandwidth, of measured", "algorithmic": alg, "traffic": None}
        tr = traffic.get(f"{wl.name}:{d['op']}")
        if tr and tr.get("kernel", "").startswith(d["kernel"]):
            r["traffic"] = tr["bytes"]
            r["traffic_source"] = tr["summary"]
        return r

    gemm_ops = detail[len(xs_shapes):]
    dom = max(gemm_ops, key=lambda d: d["ms"])
    roof = roofline_of(dom)
    rooflines = {}
    for kind, sel in (("prefill", [d for d in gemm_ops if d["bound"] == "tensor"]),
                      ("decode", [d for d in gemm_ops if d["bound"] == "hbm"]),
                      ("quantize", detail[:len(xs_shapes)])):
        if sel:
            rooflines[kind] = roofline_of(max(sel, key=lambda d: d["ms"]))

    # ---- weight quantization (load-time kernel) timed alone
    wq_ms = []
    g0 = max(wl.gemms, key=lambda g: g.N * g.K)
    for _ in range(3):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fq.fp8_quant_weight(W[g0.weight], g0.mode, out=WQ[g0.weight])
        e1.record(stream)
        torch.cuda.synchronize()
        wq_ms.append(e0.elapsed_time(e1))
    wqb = quant_bytes(g0.N, g0.K, 0) if g0.mode == 0 else (3 * g0.N * g0.K + 4 * ((g0.N + 127) // 128) * (g0.K // 128))
    weight_quant = {"shape": [g0.N, g0.K], "mode": g0.mode, "ms": round(min(wq_ms), 5),
                    "GB/s": round(wqb / (min(wq_ms) / 1e3) / 1e9, 1),
                    "frac_hbm": round(wqb / (min(wq_ms) / 1e3) / 1e9 / pk["hbm_gbs"], 3)}

    # ---- the next-step sections: each op timed like the per-op detail (R
    # back-to-back launches over R copies of its buffers, or alone when long)
    def timed(run):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
        torch.cuda._sleep(1_000_000)
        for s_ in range(args.steps):
            flush.zero_()
            ev[s_][0].record(stream)
            run()
            ev[s_][1].record(stream)
        torch.cuda.synchronize()
        return float(np.mean([a.elapsed_time(b) for a, b in ev]))

    def as_runner(fns):
        for f in fns:
            f()
        torch.cuda.synchronize()
        if args.eager:
            return lambda: [f() for f in fns]
        gr = capture(fns)
        return gr.replay

    def time_op(make, footprint):
        """(ms per launch, R, ms alone) of the op make(0); make(i) for i > 0
        builds the same op on its own copies of the op's buffers."""
        f0 = make(0)
        alone = timed(as_runner([f0]))
        if alone >= LONG_OP_MS:
            return alone, 1, alone
        R = int(min(32, max(2, -(-2 * l2_bytes // max(1, footprint)))))
        fns = [f0] + [make(i) for i in range(1, R)]
        t = timed(as_runner(fns)) / R
        del fns
        return t, R, alone

    def entry(ms, R, alone, nbytes=None, flops=None):
        e = {"ms": round(ms, 5), "back_to_back": R, "ms_isolated": round(alone, 5)}
        if nbytes is not None:
            e["GB/s"] = round(nbytes / (ms / 1e3) / 1e9, 1)
            e["frac_hbm"] = round(nbytes / (ms / 1e3) / 1e9 / pk["hbm_gbs"], 3)
        if flops is not None:
            e["TFLOP/s"] = round(flops / (ms / 1e3) / 1e12, 1)
            e["frac_fp8_peak"] = round(flops / (ms / 1e3) / 1e12 / fp8_peak, 3)
        return e

    # ---- RMSNorm + per-token quantization fused (the activations that follow
    # an RMSNorm in Llama: the inputs of q/k/v and of gate/up), next to the
    # unfused pair (torch's bf16 rms_norm, then fp8_quant_act)
    rms = []
    for k, (M, K, mode) in ([] if args.no_extras else xs_shapes.items()):
        if mode != synth.CHANNEL_TOKEN or not (k.startswith("attn_in") or k.startswith("mlp_in")):
            continue
        gmm = (1.0 + 0.1 * torch.randn(K, generator=torch.Generator().manual_seed(K))).to(torch.bfloat16).to(dev)

        def make_fused(i, k=k, gmm=gmm):
            x = X[k] if i == 0 else X[k].clone()
            o = (torch.empty_like(XQ[k][0]), torch.empty_like(XQ[k][1]))
            return lambda: fq.fp8_rmsnorm_quant_act(x, gmm, 1e-5, out=o)

        def make_unfused(i, k=k, gmm=gmm, K=K):
            x = X[k] if i == 0 else X[k].clone()
            y_n = torch.empty_like(X[k])
            o = (torch.empty_like(XQ[k][0]), torch.empty_like(XQ[k][1]))
            return lambda: (y_n.copy_(torch.nn.functional.rms_norm(x, (K,), weight=gmm, eps=1e-5)),
                            fq.fp8_quant_act(y_n, synth.CHANNEL_TOKEN, out=o))

        rb = 2 * M * K + 2 * K + M * K + 4 * M
        e = entry(*time_op(make_fused, rb), nbytes=rb)
        e.update({"act": k, "M": M, "K": K, "unfused_ms": round(time_op(make_unfused, rb + 4 * M * K)[0], 5),
                  "bytes": "2*M*K (x) + 2*K (gamma) + M*K (codes) + 4*M (scales)"})
        rms.append(e)
    assert fq.device_error(clear=True) == 0

    # ---- gate/up with the SiLU * up epilogue (one kernel, only the activation
    # written) next to the separate path: both GEMMs, then torch's silu * up
    swiglu = []
    gmap = {g.name.replace("gate_proj", "").replace("up_proj", ""): [] for g in wl.gemms}
    for g in wl.gemms:
        if g.mode == synth.CHANNEL_TOKEN and (g.name.startswith("gate_proj") or g.name.startswith("up_proj")):
            gmap[g.name.replace("gate_proj", "").replace("up_proj", "")].append(g)
    for suffix, gs in ([] if args.no_extras else gmap.items()):
        gg = [g for g in gs if g.name.startswith("gate_proj")]
        gu = [g for g in gs if g.name.startswith("up_proj")]
        if len(gg) != 1 or len(gu) != 1:
            continue
        gg, gu = gg[0], gu[0]

        def ops_of(i, gg=gg, gu=gu):
            c = (lambda t: t) if i == 0 else (lambda t: t.clone())
            return (c(XQ[gg.x][0]), c(XQ[gg.x][1]), c(WQ[gg.weight][0]), c(WQ[gg.weight][1]), c(WQ[gu.weight][0]),
                    c(WQ[gu.weight][1]))

        def make_fused(i, gg=gg):
            o = ops_of(i)
            act = torch.empty((gg.M, gg.N), dtype=torch.bfloat16, device=dev)
            return lambda: fq.fp8_linear_swiglu(*o, out=act)

        def make_separate(i, gg=gg, gu=gu):
            xq, xsc, wg, sg, wu, su = ops_of(i)
            yg = torch.empty((gg.M, gg.N), dtype=torch.bfloat16, device=dev)
            yu = torch.empty_like(yg)
            act = torch.empty_like(yg)
            wk = {g.name: (torch.zeros_like(WS[g.name]) if WS[g.name] is not None else None) for g in (gg, gu)}
            return lambda: (fq.fp8_linear(xq, xsc, wg, sg, gg.mode, out=yg, workspace=wk[gg.name]),
                            fq.fp8_linear(xq, xsc, wu, su, gu.mode, out=yu, workspace=wk[gu.name]),
                            torch.mul(torch.nn.functional.silu(yg), yu, out=act))

        fl = 2 * gg.flops
        fb = gg.M * gg.K + 2 * gg.N * gg.K + 2 * gg.M * gg.N
        e = entry(*time_op(make_fused, fb), flops=fl)
        e.update({"gemms": f"{gg.name}+{gu.name}:{gg.M}x{gg.K}->{gg.N}",
                  "separate_ms": round(time_op(make_separate, fb + 4 * gg.M * gg.N)[0], 5),
                  "note": "fused: one kernel writes bf16(bf16(silu(gate)) * up); separate: two GEMMs "
                          "writing gate and up, then torch silu and mul"})
        swiglu.append(e)
    assert fq.device_error(clear=True) == 0

    # ---- static-scale quantization (offline-calibrated scale, no amax pass)
    qstatic = []
    for k, (M, K, mode) in ([] if args.no_extras else xs_shapes.items()):
        if mode != synth.CHANNEL_TOKEN:
            continue
        sc = fq.calibrate_static_scale(X[k][: min(M, 256)])

        def make(i, k=k, sc=sc):
            x = X[k] if i == 0 else X[k].clone()
            o = (torch.empty_like(XQ[k][0]), torch.empty_like(XQ[k][1]))
            return lambda: fq.fp8_quant_act_static(x, sc, out=o)

        qb = 3 * M * K + 4 * M
        e = entry(*time_op(make, qb), nbytes=qb)
        e.update({"act": k, "M": M, "K": K})
        qstatic.append(e)
    assert fq.device_error(clear=True) == 0

    # ---- FP8 KV cache: the k_proj / v_proj outputs quantized per (token, head)
    kvq = []
    for g in ([] if args.no_extras else wl.gemms):
        if g.name not in ("k_proj", "v_proj") or g.N % 128:
            continue

        def make(i, g=g):
            kv = (Y[g.name] if i == 0 else Y[g.name].clone()).view(g.M, g.N // 128, 128)
            o = (torch.empty(kv.shape, dtype=torch.uint8, device=dev),
                 torch.empty((g.M, g.N // 128), dtype=torch.float32, device=dev))
            return lambda: fq.fp8_quant_kv(kv, out=o)

        kb = 3 * g.M * g.N + 4 * g.M * (g.N // 128)
        e = entry(*time_op(make, kb), nbytes=kb)
        e.update({"kv": g.name, "tokens": g.M, "heads": g.N // 128})
        kvq.append(e)
    assert fq.device_error(clear=True) == 0

    # ---- weight-only FP8 (bf16 activations, codes widened in the kernel):
    # the decode GEMMs (M <= 64, channel scales), next to the W8A8 path
    # (activation quantization + FP8 linear) on the same layer
    w8a16 = []
    for g in ([] if args.no_extras else wl.gemms):
        if g.mode != synth.CHANNEL_TOKEN or g.M > 64:
            continue

        def make16(i, g=g):
            x = X[g.x] if i == 0 else X[g.x].clone()
            wq = WQ[g.weight][0] if i == 0 else WQ[g.weight][0].clone()
            y16 = torch.empty((g.M, g.N), dtype=torch.bfloat16, device=dev)
            wk16 = torch.zeros(max(16, fq.fp8_linear_w8a16_workspace_size(g.M, g.N, g.K)), dtype=torch.uint8,
                               device=dev)
            return lambda: fq.fp8_linear_w8a16(x, wq, WQ[g.weight][1], out=y16, workspace=wk16)

        def make8(i, g=g):
            x = X[g.x] if i == 0 else X[g.x].clone()
            wq = WQ[g.weight][0] if i == 0 else WQ[g.weight][0].clone()
            y16 = torch.empty((g.M, g.N), dtype=torch.bfloat16, device=dev)
            xq_w, xs_w = torch.empty_like(XQ[g.x][0]), torch.empty_like(XQ[g.x][1])
            wk = torch.zeros_like(WS[g.name])
            return lambda: (fq.fp8_quant_act(x, g.mode, out=(xq_w, xs_w)),
                            fq.fp8_linear(xq_w, xs_w, wq, WQ[g.weight][1], g.mode, out=y16, workspace=wk))

        wb = g.N * g.K + 2 * g.M * g.K + 4 * g.N + 2 * g.M * g.N
        e = entry(*time_op(make16, wb), nbytes=wb)
        e.update({"gemm": g.name, "M": g.M, "N": g.N, "K": g.K, "w8a8_ms": round(time_op(make8, wb)[0], 5),
                  "kernel": "cuda cores" if g.M == 1 else "tcgen05 bf16 (widened tiles)"})
        w8a16.append(e)
    assert fq.device_error(clear=True) == 0

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        Xh = {k: X[k].cpu().pin_memory() for k in X}
        Yh = {g.name: torch.empty((g.M, g.N), dtype=torch.bfloat16).pin_memory() for g in wl.gemms}
        Xd = {k: torch.empty_like(X[k]) for k in X}

        def e2e_step():
            for k in X:
                Xd[k].copy_(Xh[k], non_blocking=True)
            for k, (M, K, mode) in xs_shapes.items():
                fq.fp8_quant_act(Xd[k], mode, out=XQ[k])
            for g in wl.gemms:
                xq, xsc = XQ[g.x]
                wq, wsc = WQ[g.weight]
                fq.fp8_linear(xq, xsc, wq, wsc, g.mode, out=Y[g.name], workspace=WS[g.name])
                Yh[g.name].copy_(Y[g.name], non_blocking=True)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        e_ms = []
        for _ in range(args.steps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step()
            b.record(stream)
            e_ms.append((a, b))
        torch.cuda.synchronize()
        barrier(world)
        et = max_over_ranks(sum(a.elapsed_time(b) for a, b in e_ms) / 1e3, world)
        e2e = {"value": round(to_metric(sum_over_ranks(units, world), et, unit), 3), "unit": unit,
               "h2d_bytes_per_step": int(sum(x.numel() * 2 for x in X.values())),
               "d2h_bytes_per_step": int(sum(y.numel() * 2 for y in Y.values())),
               "ms_per_step": round(et * 1e3 / args.steps, 4),
               "path": "pinned host X -> device, fp8_quant_act, fp8_linear, device Y -> pinned host"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, unit, args.cpu_sample_rows)

    if rank == 0:
        line = {
            "metric": metric, "value": round(value, 3), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total_s * 1e3 / args.steps, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3 (fp32 accumulate, bf16 out)", "data": "synthetic",
            "config": config_of(wl, world, args.flush_mib),
            "launch": "eager" if args.eager else
            "step: one CUDA graph replayed per step; per-op detail (and rooflines): ms = one graph of R "
            "back-to-back launches of the op over R copies of its buffers (R = back_to_back, footprint >= 2x L2, "
            "so every launch reads from DRAM) / R, after an L2 flush; ms_isolated = one launch in its own graph "
            "after an L2 flush, which ms reports (back_to_back = 1) for ops of 0.25 ms or more",
            "roofline": roof, "rooflines": rooflines, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * launches_per_step,
            "gpu_launches_source": launches_source,
            "clocks": dict(clk.summary(), measured=mon.summary()), "detail": detail, "weight_quant": weight_quant, "rmsnorm_quant": rms, "kv_quant": kvq, "swiglu": swiglu, "quant_static": qstatic, "w8a16": w8a16,
            "merged_shared_input": merged,
            "device_error": err, "gpu": torch.cuda.get_device_name(dev),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


# ----------------------------------------------------------- CPU oracle ---

def oracle_sample(wl, rows, w_cache=None):
    """Run the oracle on `rows` rows of every GEMM (all N, all K), after its
    activation quantization; returns (seconds, weight cache).  Weights are
    quantized by the oracle once, before timing, as in the GPU step."""
    import oracle
    oracle.build()
    if w_cache is None:
        w_cache = {}
    for g in wl.gemms:
        if g.weight not in w_cache:
            w = synth.make_w(g.N, g.K, seed=synth.weight_seed(g.weight))
            w_cache[g.weight] = oracle.quant_weight(w, g.mode)
    xs = {}
    for g in wl.gemms:
        if g.x not in xs:
            xs[g.x] = synth.make_x(min(rows, g.M), g.K, seed=7)
    t0 = time.perf_counter()
    q = {}
    for g in wl.gemms:
        if g.x not in q:
            q[g.x] = oracle.quant_act(xs[g.x], g.mode)
    for g in wl.gemms:
        xq, xsc = q[g.x]
        wq, wsc = w_cache[g.weight]
        oracle.linear(xq, xsc, wq, wsc, g.mode)
    return time.perf_counter() - t0, w_cache


def sample_workload(wl, rows):
    """The workload with every GEMM cut to its first `rows` token rows."""
    return synth.Workload(wl.name, [dataclasses.replace(g, M=min(rows, g.M)) for g in wl.gemms])


def omp_threads():
    n = os.environ.get("OMP_NUM_THREADS")
    if n and n.isdigit():
        return int(n)
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, unit, rows, w_cache=None, target_s=10.0):
    """The oracle on the host cores, timed over a bounded sample of the
    workload: the first `rows` token rows of every GEMM (all N, all K),
    grown (up to each GEMM's M) while one pass takes well under target_s,
    then passes repeated until about target_s of CPU work.  The value is the
    sample's own work (in the metric's unit) over its own time."""
    secs, w_cache = oracle_sample(wl, rows, w_cache)
    max_m = max(g.M for g in wl.gemms)
    while secs < target_s / 3 and rows < max_m:
        rows = min(max_m, max(2 * rows, int(rows * target_s / 3 / max(secs, 1e-3))))
        secs, w_cache = oracle_sample(wl, rows, w_cache)
    total, passes = secs, 1
    while total < target_s:
        s_, _ = oracle_sample(wl, rows, w_cache)
        total += s_
        passes += 1
    whole = all(rows >= g.M for g in wl.gemms)
    units = step_units(sample_workload(wl, rows), unit) * passes
    return {"value": round(to_metric(units, total, unit), 6), "unit": unit,
            "cores": omp_threads(), "kind": "oracle",
            "sample": (f"{'all' if whole else f'the first {rows}'} token rows of every GEMM (all N, all K): "
                       f"activation quantization + exact int64 GEMM, {passes} passes, {total:.1f} s of CPU work; "
                       "value = the sample's work over its time (weights quantized before timing, as in the GPU "
                       "step)")}


def run_reference(args):
    """The reference arm: the CPU oracle, timed step by step.  A step is the
    oracle on a bounded sample of the workload (the first --ref-sample-rows
    token rows of every GEMM, all N and all K, with their activation
    quantization); ms_per_step is that sampled step's measured time and value
    the sample's work over it."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    wl = select(args)
    metric, unit = metric_for(wl)
    rows = args.ref_sample_rows
    cache = {}
    oracle_sample(wl, 1, cache)                      # weights quantized once, before timing
    for _ in range(args.warmup):
        oracle_sample(wl, rows, cache)
    secs = [oracle_sample(wl, rows, cache)[0] for _ in range(args.steps)]
    units = step_units(sample_workload(wl, rows), unit) * args.steps
    value = to_metric(units, sum(secs), unit)
    sample = (f"each step: the first {rows} token rows of every GEMM (all N, all K), activation quantization "
              "+ exact int64 GEMM on the host cores; value = the sampled steps' work over their measured time")
    line = {"impl": "reference", "metric": metric, "value": round(value, 6), "unit": unit,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(sum(secs) * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int64 exact dot products, f64 scaling", "data": "synthetic",
            "config": config_of(wl, world, args.flush_mib),
            "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": omp_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
