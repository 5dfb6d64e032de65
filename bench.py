"""Benchmark of the weight-quantized linear layer on B200.

One JSON line on rank 0.  A "step" is one pass of the hot path over one
batch of synthetic input: for the headline workload (single-stream MTP4
verify chunk, M = 5 = 1 + 4 drafted tokens) that is the three INT4 layers
5120->5120, 5120->17408 and 17408->5120 (group 128), each a w4a16_gemm
through the C ABI.  Weights are re-packed once, outside the timed region.

value      weight-stream TB/s of the headline workload: (code + scale bytes
           of every layer in the step) / device time per step, whole job
           (all ranks).  Tensor-bound workloads are in TFLOP/s (2*M*N*K).
configs    the other measured configurations, each timed the same way on
           its own rotating weight pool: the tiny INT4 layer, the C32 MTP3
           chunk (M = 128), the prefill chunk (M = 8192) and MXFP8 at M = 4
           and M = 128 (default), with value, time per step, median / p10 /
           p90 over the steps, the in-step time of every layer and the
           roofline fractions.
e2e        the same metric through the public API with host buffers: per
           step the host-to-device copy of the step's X from pinned memory,
           the layers (prepared calls: arguments marshalled once per layer
           and pool slot, as a serving loop does; e2e_plain: the plain calls
           that check every buffer each time), the device-to-host copy of
           every Y, then a stream synchronize, timed on the host clock (e2e_graph: the same steps
           captured as CUDA graphs over consecutive pool slots and replayed,
           as a serving loop does, timed with device events).
timing     exactly --steps steps, replayed from CUDA graphs of up to 16
           consecutive steps on consecutive slots of the weight pool (the
           launches overlap their neighbours through programmatic dependent
           launch inside a replay), CUDA events on the launch stream;
           median / p10 / p90 over the replays (ms per step).
roofline   every layer of a step runs the same kernel, so the dominant
           kernel's time inside the step is the step time (its layers'
           in-step times add up to it exactly: each layer's share is the
           difference between the step cut after that layer and the step
           cut before it, both timed as graphs with the same PDL overlap);
           achieved = algorithmic bytes (or flops) per step / step time,
           against MEASURED_PEAKS.json.  The same kernels timed one launch
           at a time (no overlap with a neighbour) are reported beside it.
L2         every step reads a different copy of the weights from a rotating
           pool of at least 3 x L2 bytes, so weights come from HBM.
m_sweep    informational: the INT4 5120 -> 17408 layer at M = 1 .. 8192 on
           the path the library picks, time per layer and the fraction of
           max(bytes / HBM peak, flops / bf16 burst peak) (--no-sweep skips).

--impl reference runs the fp64 CPU oracle (the baseline arm) on the same
workload: each step processes a bounded slice of columns of every layer, and
the value is scaled by the bytes that slice covers.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

METRIC = "W4A16/MXFP8 GEMM weight-stream TB/s and TFLOP/s vs roofline, M=1..8192"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# workload -> (format, M, [(K, N)], group)
WORKLOADS = {
    "mtp4_verify_int4": ("int4", 5, [(5120, 5120), (5120, 17408), (17408, 5120)], 128),
    # the same step with the MLP gate and up projections fused into one
    # 5120 -> 34816 layer (two 17408-column parts in one re-packed buffer)
    "mtp4_verify_int4_fused": ("int4", 5, [(5120, 5120), (5120, 34816), (17408, 5120)], 128),
    "tiny_int4": ("int4", 1, [(512, 512)], 128),
    "c32_mtp3_int4": ("int4", 128, [(5120, 17408), (17408, 5120)], 128),
    "prefill_int4": ("int4", 8192, [(5120, 17408)], 128),
    "mxfp8_m4": ("mxfp8", 4, [(5120, 17408)], 32),
    "mxfp8_m128": ("mxfp8", 128, [(5120, 17408)], 32),
    # the INT8 vocabulary head (248 k columns) at the verify chunk of one stream
    "head_int8_m5": ("int8", 5, [(5120, 248320)], 128),
    # the paired dense bf16 GDN A/B projection (2 x 48 rows of 5120)
    "gdn_ab_bf16_m4": ("bf16", 4, [(5120, 96)], 0),
    "gdn_ab_bf16_m1": ("bf16", 1, [(5120, 96)], 0),
}
TENSOR_BOUND = {"c32_mtp3_int4", "prefill_int4", "mxfp8_m128"}
# both fractions are reported for these (the ridge regime)
BOTH_FRACTIONS = {"c32_mtp3_int4", "mxfp8_m128"}
# (workload, layer index) -> column counts of the projections fused into it
FUSED_PARTS = {("mtp4_verify_int4_fused", 1): (17408, 17408)}
# the five measured configurations besides nothing else: the headline first
DEFAULT_CONFIGS = ["mtp4_verify_int4", "tiny_int4", "c32_mtp3_int4", "prefill_int4",
                   "mxfp8_m4", "mxfp8_m128"]
# at least this many timed steps for a secondary configuration (its timed
# region stays above a millisecond or so); the headline times exactly --steps
MIN_STEPS = {"tiny_int4": 400, "mtp4_verify_int4": 200, "mtp4_verify_int4_fused": 200,
             "c32_mtp3_int4": 100, "prefill_int4": 10, "mxfp8_m4": 200, "mxfp8_m128": 100,
             "head_int8_m5": 20, "gdn_ab_bf16_m4": 400, "gdn_ab_bf16_m1": 400}
# MXFP8 at M <= 16 runs on the re-packed layout (mxfp8_repack, once, outside
# the timed region) through mxfp8_gemm_packed; larger M on the stored layout
MXFP8_PACKED_MAX_M = 16
KERNELS = {"bf16": "bf16_small_kernel", "int4": "w4a16_stream_kernel",
           "int8": "w4a16_stream_kernel", "mxfp8": "mxfp8_stream_kernel"}


def layer_weight_bytes(fmt, K, N, G):
    if fmt == "int4":
        return N * K // 2 + N * (K // G) * 2
    if fmt == "bf16":
        return N * K * 2
    if fmt == "int8":
        return N * K + N * (K // G) * 2
    return N * K + N * (K // 32)


def kernel_of(fmt, M):
    if fmt in ("int4", "mxfp8") and M > 32:
        return "tc_gemm_kernel"
    if fmt == "mxfp8" and M <= MXFP8_PACKED_MAX_M:
        return "w4a16_stream_kernel"   # the re-packed MXFP8 variant of the weight stream
    return KERNELS[fmt]


def arith_dtype(fmt, M):
    """Operand type of the tensor-core products of a workload: the INT4 and
    INT8 weight streams at M <= 16 multiply fp16 operands (codes decoded
    exactly to 1024 + q or 1024 + 16 q, activations scaled per group by a
    power of two into fp16 exactly); every other path multiplies bf16
    operands.  Accumulation is fp32 throughout."""
    return "f16" if fmt in ("int4", "int8", "mxfp8") and M <= 16 else "bf16"


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def quantiles(xs):
    """(median, p10, p90) of a list of numbers."""
    a = np.asarray(xs, dtype=np.float64)
    return (float(np.median(a)), float(np.percentile(a, 10)), float(np.percentile(a, 90)))


# --------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        # the raw samples (the JSON line carries their summary); MXG_CLOCKS_DIR
        # keeps them somewhere else than the system temporary directory
        base = os.environ.get("MXG_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(base, f"mxg_clocks_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                except ValueError:
                    continue
                for name, v in zip(names, parts[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "samples": len(sm), "reasons": sorted(reasons)}


def max_over_ranks(x: float, world: int, device) -> float:
    """The job's time is the slowest rank's: MAX all-reduce of one number
    (the NCCL group on GPUs; any initialised group, e.g. gloo, on CPU)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_rank: float, world: int, elapsed_max_ms: float) -> float:
    """Whole-job throughput (weak scaling): every rank processed the same
    units, the job took the slowest rank's time."""
    return world * units_per_rank / (elapsed_max_ms * 1e-3)


# ------------------------------------------------------------------ our arm
class Workload:
    """Seeded inputs of one workload on one device: per layer a rotating pool
    of weight copies (>= pool_factor x L2 bytes per step), X, Y and a
    workspace, and the library call of each layer."""

    def __init__(self, name, rank, dev, pool_factor):
        import torch

        import mxfp8_gemm_speculative_b200 as mxg
        import synth
        self.mxg, self.name, self.dev = mxg, name, dev
        self.fmt, self.M, self.layers, self.G = WORKLOADS[name]
        fmt, M, G = self.fmt, self.M, self.G
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.step_bytes = sum(layer_weight_bytes(fmt, K, N, G) for K, N in self.layers)
        self.step_flops = sum(2 * M * N * K for K, N in self.layers)
        self.pool = max(2, -(-int(pool_factor * l2) // self.step_bytes))
        self.xs, self.ys, self.weights, self.wss = [], [], [], []
        for li, (K, N) in enumerate(self.layers):
            if fmt == "int4":
                lay = synth.int4_layer(M, K, N, G, seed=rank, layer=li)
                qw = torch.from_numpy(lay.qweight).to(dev)
                sc = torch.from_numpy(lay.scales.view(np.int16)).to(dev)
                parts = FUSED_PARTS.get((name, li))
                if parts:
                    # fused projections: the parts' columns of the seeded layer,
                    # re-packed into one buffer
                    bounds = np.cumsum((0,) + parts)
                    packed = mxg.w4a16_repack_fused(
                        [(qw[:, a:b].contiguous(), sc[:, a:b].contiguous())
                         for a, b in zip(bounds[:-1], bounds[1:])], G)
                else:
                    packed = mxg.w4a16_repack(qw, sc, G)
                del qw, sc
                self.weights.append([packed] + [packed.clone() for _ in range(self.pool - 1)])
                need = mxg.w4a16_workspace_bytes(M, N, K, G)
            elif fmt == "int8":
                lay = synth.int8_layer(M, K, N, G, seed=rank, layer=li)
                qw = torch.from_numpy(lay.qweight).to(dev)
                sc = torch.from_numpy(lay.scales.view(np.int16)).to(dev)
                packed = mxg.w8a16_repack(qw, sc, G)
                del qw, sc
                self.weights.append([packed] + [packed.clone() for _ in range(self.pool - 1)])
                need = mxg.raw_lib().w8a16_workspace_bytes(M, N, K, G)
            elif fmt == "bf16":
                lay = synth.bf16_layer(M, K, N, seed=rank, layer=li)
                w = torch.from_numpy(lay.W.view(np.int16)).view(torch.bfloat16).to(dev)
                self.weights.append([w] + [w.clone() for _ in range(self.pool - 1)])
                need = mxg.raw_lib().bf16_gemm_small_workspace_bytes(M, N, K)
            else:
                lay = synth.mxfp8_layer(M, K, N, seed=rank, layer=li)
                wq = torch.from_numpy(lay.Wq).to(dev)
                ws = torch.from_numpy(lay.Ws).to(dev)
                if M <= MXFP8_PACKED_MAX_M:
                    packed = mxg.mxfp8_repack(wq, ws)
                    del wq, ws
                    self.weights.append([packed] + [packed.clone() for _ in range(self.pool - 1)])
                    need = mxg.mxfp8_packed_workspace_bytes(M, N, K)
                else:
                    self.weights.append([(wq, ws)] + [(wq.clone(), ws.clone())
                                                      for _ in range(self.pool - 1)])
                    need = mxg.mxfp8_workspace_bytes(M, N, K)
            self.wss.append(torch.zeros(need, dtype=torch.uint8, device=dev))
            self.xs.append(torch.from_numpy(lay.X.view(np.int16)).view(torch.bfloat16).to(dev))
            self.ys.append(torch.empty((M, N), dtype=torch.bfloat16, device=dev))
        self.kernel = kernel_of(fmt, M)

    def round_pool(self, seg):
        """Grow the weight pool to a multiple of `seg` slots (more copies of
        the same weights), so graphs of `seg` steps tile it exactly."""
        while self.pool % seg:
            for w in self.weights:
                w.append(w[0].clone() if not isinstance(w[0], tuple)
                         else tuple(t.clone() for t in w[0]))
            self.pool += 1

    def prepare(self, li, p, s, x, y):
        """Layer li on pool slot p as a prepared call of the public API
        (arguments marshalled once, as a serving loop does)."""
        mxg, fmt, G = self.mxg, self.fmt, self.G
        K, N = self.layers[li]
        w = self.weights[li][p]
        kw = dict(out=y, workspace_buf=self.wss[li], stream=s)
        if fmt == "int4":
            return mxg.prepare_w4a16_gemm(x, w, N, K, G, **kw)[0]
        if fmt == "int8":
            return mxg.prepare_w8a16_gemm(x, w, N, K, G, **kw)[0]
        if fmt == "bf16":
            return mxg.prepare_bf16_gemm_small(x, w, **kw)[0]
        if self.M <= MXFP8_PACKED_MAX_M:
            return mxg.prepare_mxfp8_gemm_packed(x, w, N, K, **kw)[0]
        return mxg.prepare_mxfp8_gemm(x, w[0], w[1], **kw)[0]

    def call(self, li, p, s, x=None, y=None):
        """Layer li on pool slot p, on stream s (X and Y default to the
        workload's device buffers)."""
        mxg, fmt, G = self.mxg, self.fmt, self.G
        K, N = self.layers[li]
        x = self.xs[li] if x is None else x
        y = self.ys[li] if y is None else y
        w = self.weights[li][p]
        if fmt == "int4":
            mxg.w4a16_gemm(x, w, N, K, G, out=y, workspace_buf=self.wss[li], stream=s)
        elif fmt == "int8":
            mxg.w8a16_gemm(x, w, N, K, G, out=y, workspace_buf=self.wss[li], stream=s)
        elif fmt == "bf16":
            mxg.bf16_gemm_small(x, w, out=y, workspace_buf=self.wss[li], stream=s)
        elif self.M <= MXFP8_PACKED_MAX_M:
            mxg.mxfp8_gemm_packed(x, w, N, K, out=y, workspace_buf=self.wss[li], stream=s)
        else:
            mxg.mxfp8_gemm(x, w[0], w[1], out=y, workspace_buf=self.wss[li], stream=s)

    def status(self):
        return max(abs(self.mxg.mxg_workspace_status(w)) for w in self.wss)


def capture(torch, stream, fn):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def segment_len(steps: int, pool: int) -> int:
    """Steps per captured graph: the largest divisor of `steps` that is at
    most min(pool, 16), so the timed region is whole replays."""
    cap = max(1, min(pool, 16))
    return max(d for d in range(1, cap + 1) if steps % d == 0)


def time_segments(torch, stream, graphs, steps, seg, per_replay_events):
    """Device time of exactly `steps` steps replayed as `steps // seg` graph
    replays, graph i % len(graphs) at replay i (the graphs hold consecutive
    runs of `seg` pool slots, so the replays walk the pool in order).  With
    per_replay_events, an event between replays gives the ms per step of
    every replay."""
    n = steps // seg
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1 if per_replay_events else 2)]
    with torch.cuda.stream(stream):
        evs[0].record(stream)
        for i in range(n):
            graphs[i % len(graphs)].replay()
            if per_replay_events:
                evs[i + 1].record(stream)
        if not per_replay_events:
            evs[1].record(stream)
    torch.cuda.synchronize()
    total = evs[0].elapsed_time(evs[-1])
    per = ([evs[i].elapsed_time(evs[i + 1]) / seg for i in range(n)] if per_replay_events else [])
    return total, per


def isolated_launch_us(torch, wl, stream, launches):
    """Each layer timed one launch at a time: an event pair around every
    launch, the launches queued behind a sleep kernel so every pair brackets
    exactly one kernel (no overlap with a neighbour)."""
    nl = len(wl.layers)
    acc = [0.0] * nl
    done = 0
    with torch.cuda.stream(stream):
        while done < launches:
            nb = min(64, launches - done)
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * nl * nb)]
            torch.cuda._sleep(20_000_000)
            for i in range(nb):
                p = (done + i) % wl.pool
                for li in range(nl):
                    evs[2 * (i * nl + li)].record(stream)
                    wl.call(li, p, stream)
                    evs[2 * (i * nl + li) + 1].record(stream)
            torch.cuda.synchronize()
            for i in range(nb):
                for li in range(nl):
                    acc[li] += evs[2 * (i * nl + li)].elapsed_time(evs[2 * (i * nl + li) + 1])
            done += nb
    return [a / launches * 1e3 for a in acc]


def measure(wl, steps, warmup, world, dev, args, with_e2e):
    """Times one workload: exactly `steps` steps after `warmup`, replayed
    from CUDA graphs of `seg` consecutive steps on consecutive weight-pool
    slots (a serving loop's graph of consecutive layers: the launches overlap
    their neighbours through programmatic dependent launch, within a replay
    and not across the replay boundary); per-replay quantiles; in-step
    per-layer times; one-launch-at-a-time kernel times; the e2e figures."""
    import torch
    import torch.distributed as dist

    stream = torch.cuda.Stream(dev)
    nl = len(wl.layers)
    seg = segment_len(steps, wl.pool)
    wl.round_pool(seg)
    nseg = wl.pool // seg

    def graphs_for(j):
        # the pool's segments, each step cut after layer j (j = nl: whole steps)
        return [capture(torch, stream, lambda o=o: [wl.call(li, p, stream)
                                                    for p in range(o, o + seg)
                                                    for li in range(j)])
                for o in range(0, wl.pool, seg)]

    with torch.cuda.stream(stream):
        for li in range(nl):
            wl.call(li, 0, stream)          # plans and kernel attributes outside capture
        torch.cuda.synchronize(dev)
        graphs = {j: graphs_for(j) for j in range(1, nl + 1)}
    with torch.cuda.stream(stream):
        for i in range(max(nseg, -(-warmup // seg))):
            graphs[nl][i % nseg].replay()
    torch.cuda.synchronize(dev)
    status = wl.status()
    if status:
        raise RuntimeError(f"{wl.name}: kernel reported status {-status}")
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    elapsed_ms, _ = time_segments(torch, stream, graphs[nl], steps, seg, False)
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    # the distribution over replays (an event between replays), same steps
    _, per_step = time_segments(torch, stream, graphs[nl], steps, seg, True)
    # in-step share of every layer: steps cut after layer j minus steps cut
    # after layer j - 1
    in_step = []
    if nl > 1:
        prev = 0.0
        for j in range(1, nl + 1):
            t, _ = time_segments(torch, stream, graphs[j], steps, seg, False)
            in_step.append((t - prev) / steps * 1e3)
            prev = t
        # rescale so the shares add up to the whole-step time measured above
        scale = (elapsed_ms / steps * 1e3) / max(sum(in_step), 1e-9)
        in_step = [v * scale for v in in_step]
    else:
        in_step = [elapsed_ms / steps * 1e3]
    iso = isolated_launch_us(torch, wl, stream, max(wl.pool, min(steps, args.kernel_steps)))
    if wl.status():
        raise RuntimeError(f"{wl.name}: kernel reported a status")
    res = {"elapsed_ms": elapsed_ms, "per_step_ms": per_step, "in_step_us": in_step,
           "isolated_us": iso, "cycle_steps": seg}
    if with_e2e:
        res.update(measure_e2e(wl, stream, steps, world, dev, args, seg))
    del graphs
    return res


def measure_e2e(wl, stream, steps, world, dev, args, seg):
    """End to end through the public API with host buffers."""
    import torch
    import torch.distributed as dist

    e2e_steps = max(1, min(args.e2e_steps, max(steps, 1)))
    x_sizes = [x.numel() for x in wl.xs]
    y_sizes = [y.numel() for y in wl.ys]
    host_x = torch.cat([x.reshape(-1).cpu() for x in wl.xs]).pin_memory()
    host_y = torch.empty(sum(y_sizes), dtype=torch.bfloat16).pin_memory()
    dev_xbuf = torch.empty(sum(x_sizes), dtype=torch.bfloat16, device=dev)
    dev_ybuf = torch.empty(sum(y_sizes), dtype=torch.bfloat16, device=dev)
    dev_x = [v.view(x.shape) for v, x in zip(torch.split(dev_xbuf, x_sizes), wl.xs)]
    dev_y = [v.view(y.shape) for v, y in zip(torch.split(dev_ybuf, y_sizes), wl.ys)]
    h2d, d2h = host_x.numel() * 2, host_y.numel() * 2
    nl = len(wl.layers)

    def step(p):
        dev_xbuf.copy_(host_x, non_blocking=True)
        for li in range(nl):
            wl.call(li, p, stream, x=dev_x[li], y=dev_y[li])
        host_y.copy_(dev_ybuf, non_blocking=True)

    prepared = {(li, p): wl.prepare(li, p, stream, dev_x[li], dev_y[li])
                for p in range(min(wl.pool, e2e_steps)) for li in range(nl)}

    def step_prepared(p):
        dev_xbuf.copy_(host_x, non_blocking=True)
        for li in range(nl):
            prepared[(li, p)]()
        host_y.copy_(dev_ybuf, non_blocking=True)

    def eager(fn, slots):
        # what a Python caller of the public API sees, host clock
        with torch.cuda.stream(stream):
            for i in range(3):
                fn(i % slots)
            stream.synchronize()
            if world > 1:
                dist.barrier()
            t0 = time.perf_counter()
            for i in range(e2e_steps):
                fn(i % slots)
                stream.synchronize()            # the result is on the host
            ms = (time.perf_counter() - t0) * 1e3
        return max_over_ranks(ms, world, dev)

    # (1) prepared calls (marshalled once per layer and slot), (1b) plain calls
    eager_ms = eager(step_prepared, min(wl.pool, e2e_steps))
    plain_ms = eager(step, wl.pool)
    del prepared
    # (2) the steps captured as graphs of `seg` consecutive pool slots and
    # replayed, device events
    eseg = segment_len(e2e_steps, seg)
    with torch.cuda.stream(stream):
        graphs = [capture(torch, stream, lambda o=o: [step(p) for p in range(o, o + eseg)])
                  for o in range(0, wl.pool - eseg + 1, eseg)]
        graphs[0].replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    graph_ms, _ = time_segments(torch, stream, graphs, e2e_steps, eseg, False)
    graph_ms = max_over_ranks(graph_ms, world, dev)
    del graphs
    return {"e2e_steps": e2e_steps, "e2e_eager_ms": eager_ms, "e2e_plain_ms": plain_ms,
            "e2e_graph_ms": graph_ms, "h2d": h2d, "d2h": d2h}


def summarize(wl, res, steps, world, peaks, peak_kind):
    """The measured numbers of one workload as a JSON-able dict."""
    tensor_bound = wl.name in TENSOR_BOUND
    elapsed_ms = res["elapsed_ms"]
    ms_per_step = elapsed_ms / steps
    if tensor_bound:
        unit = "TFLOP/s"
        value = job_value(wl.step_flops * steps, world, elapsed_ms) / 1e12
    else:
        unit = "TB/s"
        value = job_value(wl.step_bytes * steps, world, elapsed_ms) / 1e12
    med, p10, p90 = quantiles(res["per_step_ms"]) if res["per_step_ms"] else (None,) * 3
    # in-step time of the dominant kernel = every layer of the step
    k_us = sum(res["in_step_us"])
    hbm_gbs = wl.step_bytes / (k_us * 1e-6) / 1e9
    tflops = wl.step_flops / (k_us * 1e-6) / 1e12
    if tensor_bound:
        # the sustained peak (a seconds-long cuBLAS loop under the power cap)
        # for a timed region of back-to-back GEMMs longer than 0.1 s, the
        # burst peak otherwise; both fractions are reported
        sustained = elapsed_ms > 100.0
        pk = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(tflops, 2), "peak": pk,
                "unit": "TFLOP/s", "frac": round(tflops / pk, 4),
                "peak_source": (f"{peak_kind} bf16 dense, sustained (timed region "
                                f"{elapsed_ms / 1e3:.2f} s of back-to-back GEMMs)" if sustained
                                else f"{peak_kind} bf16 dense (burst)"),
                "frac_of_burst": round(tflops / peaks["bf16_tflops"], 4),
                "frac_of_sustained": round(tflops / peaks["bf16_tflops_sustained"], 4)}
    else:
        roof = {"bound": "hbm", "achieved": round(hbm_gbs, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(hbm_gbs / peaks["hbm_gbs"], 4),
                "peak_source": f"{peak_kind} copy bandwidth"}
    if wl.name in BOTH_FRACTIONS:
        roof["fractions"] = {"hbm": round(hbm_gbs / peaks["hbm_gbs"], 4),
                             "tensor": round(tflops / peaks["bf16_tflops"], 4),
                             "hbm_gbs": round(hbm_gbs, 1), "tflops": round(tflops, 2)}
    roof["traffic"] = traffic_from_profiles(wl.kernel, wl.name)
    roof["kernel"] = wl.kernel
    roof["in_step_us_per_layer"] = [round(v, 3) for v in res["in_step_us"]]
    roof["isolated_us_per_layer"] = [round(v, 3) for v in res["isolated_us"]]
    iso_us = sum(res["isolated_us"])
    roof["isolated_achieved"] = round(
        (wl.step_flops / (iso_us * 1e-6) / 1e12) if tensor_bound
        else (wl.step_bytes / (iso_us * 1e-6) / 1e9), 2)
    out = {"value": round(value, 4), "unit": unit, "ms_per_step": round(ms_per_step, 6),
           "steps": steps,
           "step_ms_quantiles": {"median": med, "p10": p10, "p90": p90,
                                 "over": f"{len(res['per_step_ms'])} replays of "
                                         f"{res['cycle_steps']} steps (ms per step)"},
           "tbps": round(job_value(wl.step_bytes * steps, world, elapsed_ms) / 1e12, 4),
           "tflops": round(job_value(wl.step_flops * steps, world, elapsed_ms) / 1e12, 3),
           "roofline": roof,
           "config": {"workload": wl.name, "format": wl.fmt, "M": wl.M,
                      "dtype": arith_dtype(wl.fmt, wl.M),
                      "layers_KxN": [f"{K}x{N}" for K, N in wl.layers],
                      "group_size": (wl.G if wl.fmt in ("int4", "int8")
                                     else (32 if wl.fmt == "mxfp8" else None)),
                      "weight_bytes_per_step": wl.step_bytes, "flops_per_step": wl.step_flops,
                      "l2": f"rotating weight pool of {wl.pool} copies "
                            f"({wl.pool * wl.step_bytes / 1e6:.0f} MB per layer set)"},
           "gpu_launches": len(wl.layers) * steps}
    if "e2e_eager_ms" in res:
        n = res["e2e_steps"]
        units = (wl.step_flops if tensor_bound else wl.step_bytes) * n
        scale = 1e12
        out["e2e"] = {"value": round(job_value(units, world, res["e2e_eager_ms"]) / scale, 4),
                      "unit": unit, "h2d_bytes_per_step": res["h2d"],
                      "d2h_bytes_per_step": res["d2h"], "steps": n,
                      "path": "public Python API per step: pinned-host copy of every layer's X "
                              "in, the layer calls (prepared calls of the binding: arguments "
                              "marshalled once, each call one C-ABI call), copy of every Y out, "
                              "stream synchronize; host clock"}
        out["e2e_plain"] = {"value": round(job_value(units, world, res["e2e_plain_ms"]) / scale, 4),
                            "unit": unit, "steps": n,
                            "path": "the same with the plain binding calls (buffers checked "
                                    "every call)"}
        out["e2e_graph"] = {"value": round(job_value(units, world, res["e2e_graph_ms"]) / scale, 4),
                            "unit": unit, "steps": n,
                            "path": "the same steps captured as CUDA graphs over consecutive "
                                    "pool slots and replayed; device events"}
    return out


SWEEP_M = (1, 2, 4, 5, 8, 16, 32, 64, 128, 256, 1024, 8192)
SWEEP_LAYER = (5120, 17408)


def m_sweep(args, rank, world, dev, peaks):
    """Informational: the INT4 5120 -> 17408 layer at every M of SWEEP_M
    (the path the library picks), each timed like a configuration; time per
    layer, weight TB/s, TFLOP/s and the fraction of the layer's roofline
    time max(bytes / HBM peak, flops / burst bf16 peak)."""
    import torch

    out = []
    K, N = SWEEP_LAYER
    for M in SWEEP_M:
        name = f"sweep_int4_m{M}"
        WORKLOADS[name] = ("int4", M, [SWEEP_LAYER], 128)
        wl = Workload(name, rank, dev, args.pool_factor)
        steps = 10 if M >= 1024 else 50
        res = measure(wl, steps, 3, world, dev, args, with_e2e=False)
        us = res["elapsed_ms"] / steps * 1e3
        t_roof = max(wl.step_bytes / (peaks["hbm_gbs"] * 1e9),
                     wl.step_flops / (peaks["bf16_tflops"] * 1e12)) * 1e6
        out.append({"M": M, "us": round(us, 3),
                    "tbps": round(wl.step_bytes / (us * 1e-6) / 1e12, 4),
                    "tflops": round(wl.step_flops / (us * 1e-6) / 1e12, 2),
                    "kernel": wl.kernel, "frac_of_roofline": round(t_roof / us, 4)})
        del wl, WORKLOADS[name]
        torch.cuda.empty_cache()
    return {"layer_KxN": f"{K}x{N}", "format": "int4 g128", "points": out,
            "roofline": "max(weight bytes / measured HBM, flops / measured bf16 burst)"}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    peaks, peak_kind = load_peaks()
    names = [args.workload]
    if args.configs == "default":
        names += [n for n in DEFAULT_CONFIGS if n != args.workload]
    elif args.configs and args.configs != "none":
        names += [n for n in args.configs.split(",") if n and n != args.workload]
    for n in names:
        if n not in WORKLOADS:
            raise SystemExit(f"unknown workload {n}")

    results = {}
    for i, name in enumerate(names):
        head = i == 0
        wl = Workload(name, rank, dev, args.pool_factor)
        steps = args.steps if head else max(args.steps, MIN_STEPS.get(name, args.steps))
        warmup = args.warmup if head else max(args.warmup, 3)
        # clocks sampled while this workload is measured
        clocks = ClockSampler(local_rank)
        clocks.start()
        res = measure(wl, steps, warmup, world, dev, args, with_e2e=head or args.e2e_all)
        clk_w = clocks.stop()
        results[name] = summarize(wl, res, steps, world, peaks, peak_kind)
        results[name]["clocks"] = clk_w
        del wl
        torch.cuda.empty_cache()
    if world > 1:
        dist.barrier()
    clk = results[args.workload]["clocks"]

    head = results[args.workload]
    props = torch.cuda.get_device_properties(dev)
    line = {
        "metric": METRIC,
        "value": head["value"],
        "unit": head["unit"],
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": arith_dtype(WORKLOADS[args.workload][0], WORKLOADS[args.workload][1]),
        "data": "synthetic (seeded; the value distributions of the layer formats)",
        "config": dict(head["config"], **{
            "timing": "CUDA graphs of up to 16 consecutive steps on consecutive weight-pool "
                      "slots, replayed for exactly --steps steps, CUDA events on the launch "
                      "stream; weights from a rotating pool >= 3 x L2 (inputs larger than L2)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}),
        "step_ms_quantiles": head["step_ms_quantiles"],
        "tflops": head["tflops"],
        "tbps": head["tbps"],
        "e2e": head.get("e2e"),
        "e2e_plain": head.get("e2e_plain"),
        "e2e_graph": head.get("e2e_graph"),
        "roofline": head["roofline"],
        "gpu_launches": head["gpu_launches"],
        "clocks": clk,
        "gpu": props.name,
        "configs": {n: r for n, r in results.items() if n != args.workload},
    }
    if not args.no_sweep:
        line["m_sweep"] = m_sweep(args, rank, world, dev, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


def traffic_from_profiles(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if one matches."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d.get(workload, {}).get(kernel)
    except (OSError, ValueError):
        return None


# ------------------------------------------------------------- CPU oracle arm
def oracle_step_runner(workload: str, cols_per_layer: int | None, seed: int = 0):
    """A callable running the oracle over a column slice of every layer of the
    workload, and the weight bytes / flops that slice covers."""
    import oracle
    import synth
    fmt, M, layers, G = WORKLOADS[workload]
    prepared = []
    for li, (K, N) in enumerate(layers):
        if fmt == "int4":
            lay = synth.int4_layer(M, K, N, G, seed=seed, layer=li)
        elif fmt == "bf16":
            lay = synth.bf16_layer(M, K, N, seed=seed, layer=li)
        elif fmt == "int8":
            lay = synth.int8_layer(M, K, N, G, seed=seed, layer=li)
        else:
            lay = synth.mxfp8_layer(M, K, N, seed=seed, layer=li)
        prepared.append((K, N, lay))
    state = {"off": 0}

    def slice_inputs(K, N, lay, c0, c1):
        if fmt in ("int4", "int8"):
            return (np.ascontiguousarray(lay.qweight[:, c0:c1]),
                    np.ascontiguousarray(lay.scales[:, c0:c1]))
        if fmt == "bf16":
            return np.ascontiguousarray(lay.W[c0:c1]), None
        return (np.ascontiguousarray(lay.Wq[c0:c1]), np.ascontiguousarray(lay.Ws[c0:c1]))

    def run(nthreads: int):
        total_bytes = 0
        total_flops = 0
        for K, N, lay in prepared:
            w = N if cols_per_layer is None else min(cols_per_layer, N)
            c0 = (state["off"] * w) % N
            c1 = min(c0 + w, N)
            a, b = slice_inputs(K, N, lay, c0, c1)
            n = c1 - c0
            if fmt == "int4":
                oracle.w4a16_gemm(lay.X, a, b, M, n, K, G, nthreads=nthreads)
            elif fmt == "int8":
                oracle.w8a16_gemm(lay.X, a, b, M, n, K, G, nthreads=nthreads)
            elif fmt == "bf16":
                oracle.bf16_gemm(lay.X, a, M, n, K)
            else:
                oracle.mxfp8_gemm(lay.X, a, b, M, n, K, nthreads=nthreads)
            total_bytes += layer_weight_bytes(fmt, K, n, G)
            total_flops += 2 * M * n * K
        state["off"] += 1
        return total_bytes, total_flops

    return run, fmt


def _oracle_rate(workload: str, nthreads: int, budget_s: float):
    """(value in the workload's unit, column slice, passes, seconds) of the
    oracle on `nthreads` threads, about budget_s seconds of work."""
    fmt, M, layers, G = WORKLOADS[workload]
    probe, _ = oracle_step_runner(workload, 64)
    t0 = time.perf_counter()
    probe(nthreads)
    dt = max(time.perf_counter() - t0, 1e-6)
    full_cols = max(N for _, N in layers)
    cols = int(min(full_cols, max(16, 64 * budget_s / dt / 2)))
    run, _ = oracle_step_runner(workload, cols)
    t0 = time.perf_counter()
    b, f = run(nthreads)
    passes = 1
    while time.perf_counter() - t0 < 0.5 * budget_s:
        run(nthreads)
        passes += 1
    dt = time.perf_counter() - t0
    b, f = b * passes, f * passes
    value = (f / dt / 1e12) if workload in TENSOR_BOUND else (b / dt / 1e12)
    return value, cols, passes, dt


def cpu_baseline(workload: str, budget_s: float = 20.0):
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    used = oracle.threads(cores)
    fmt, M, layers, G = WORKLOADS[workload]
    value, cols, passes, dt = _oracle_rate(workload, used, budget_s * 0.75)
    v1, cols1, passes1, dt1 = _oracle_rate(workload, 1, budget_s * 0.25)
    unit = "TFLOP/s" if workload in TENSOR_BOUND else "TB/s"
    return {"value": value, "unit": unit, "cores": used, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": f"{cols} of the output columns of every layer of {workload} "
                      f"(M={M}), {passes} pass(es), {dt:.1f} s, fp64 C oracle, "
                      f"OpenMP over columns on {used} threads",
            "single_thread": {"value": v1, "unit": unit, "cores": 1,
                              "sample": f"{cols1} output columns of every layer, "
                                        f"{passes1} pass(es), {dt1:.1f} s"}}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    used = oracle.threads(cores)
    fmt, M, layers, G = WORKLOADS[args.workload]
    tensor_bound = args.workload in TENSOR_BOUND
    # each step: a slice of columns sized so warmup + steps end in about
    # args.ref_budget seconds
    probe, _ = oracle_step_runner(args.workload, 16)
    t0 = time.perf_counter()
    probe(used)
    dt16 = max(time.perf_counter() - t0, 1e-6)
    per_step = args.ref_budget / max(1, args.steps + args.warmup)
    cols = int(max(1, min(max(N for _, N in layers), 16 * per_step / dt16)))
    run, _ = oracle_step_runner(args.workload, cols)
    for _ in range(args.warmup):
        run(used)
    tb = tf = 0
    t0 = time.perf_counter()
    for _ in range(args.steps):
        b, f = run(used)
        tb += b
        tf += f
    dt = time.perf_counter() - t0
    value = (tf / dt / 1e12) if tensor_bound else (tb / dt / 1e12)
    unit = "TFLOP/s" if tensor_bound else "TB/s"
    sample = (f"{cols} output columns of every layer per step ({args.workload}, M={M}); "
              f"fp64 C oracle, {used} threads")
    line = {
        "impl": "reference",
        "metric": METRIC,
        "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; the value distributions of the layer formats)",
        "config": {"workload": args.workload, "format": fmt, "M": M,
                   "layers_KxN": [f"{K}x{N}" for K, N in layers]},
        "cpu_baseline": {"value": value, "unit": unit, "cores": used, "kind": "oracle",
                         "sample": sample, "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="mtp4_verify_int4",
                    help="the headline workload (the line's value)")
    ap.add_argument("--configs", default="default",
                    help="further workloads measured into the line's 'configs': 'default' "
                         "(the five configurations), 'none', or a comma list")
    ap.add_argument("--e2e-all", action="store_true",
                    help="measure the e2e figures for every configuration, not only the headline")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--kernel-steps", type=int, default=64)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the informational M sweep of the INT4 5120 -> 17408 layer")
    ap.add_argument("--pool-factor", type=float, default=3.0,
                    help="rotating weight pool size in multiples of the L2 size")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
