"""Benchmark of the weight-quantized linear layer on B200.

One JSON line on rank 0.  A "step" is one pass of the hot path over one
batch of synthetic inputs: for the default workload (single-stream MTP4
verify chunk, M = 5 = 1 + 4 drafted tokens) that is the three INT4 layers
5120->5120, 5120->17408 and 17408->5120 (group 128), each a w4a16_gemm
through the C ABI.  Weights are re-packed once, outside the timed region.

value      weight-stream TB/s: (code + scale bytes of every layer in the step)
           / device time per step, whole job (all ranks).  For tensor-bound
           workloads the line's unit is TFLOP/s (2*M*N*K per layer).
e2e        the same metric through the Python binding with host buffers:
           every step copies X from pinned host memory and reads Y back (the
           step, copies included, replayed as a CUDA graph per pool slot).
Workloads  --workload picks the step: the MTP4 verify layers (default; also
           with gate/up fused), the C32 MTP3 chunk (M = 128), a prefill chunk
           (M = 8192), MXFP8 at M = 4 and 128, the INT8 vocabulary head and
           the paired bf16 GDN A/B projection.
roofline   the dominant kernel's algorithmic bytes (or flops) per launch over
           its average launch time, timed with CUDA events on its stream,
           against MEASURED_PEAKS.json.
L2         every step reads a different copy of the weights from a rotating
           pool of at least 3 x L2 bytes, so weights come from HBM.

--impl reference runs the fp64 CPU oracle (the baseline arm) on the same
workload: each step processes a bounded slice of columns of every layer, and
the value is scaled by the bytes that slice covers.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import tempfile
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

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
# (workload, layer index) -> column counts of the projections fused into it
FUSED_PARTS = {("mtp4_verify_int4_fused", 1): (17408, 17408)}


def layer_weight_bytes(fmt, K, N, G):
    if fmt == "int4":
        return N * K // 2 + N * (K // G) * 2
    if fmt == "bf16":
        return N * K * 2
    if fmt == "int8":
        return N * K + N * (K // G) * 2
    return N * K + N * (K // 32)


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
        # samples under load: the upper half of the observed clocks
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
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import mxfp8_gemm_speculative_b200 as mxg
    import synth

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))

    fmt, M, layers, G = WORKLOADS[args.workload]
    tensor_bound = args.workload in TENSOR_BOUND
    props = torch.cuda.get_device_properties(dev)
    l2 = props.L2_cache_size

    # inputs: one seeded synthetic layer per shape (rank-dependent seed)
    step_bytes = sum(layer_weight_bytes(fmt, K, N, G) for K, N in layers)
    step_flops = sum(2 * M * N * K for K, N in layers)
    pool = max(2, -(-int(args.pool_factor * l2) // step_bytes))
    xs, ys, weights, wss = [], [], [], []
    for li, (K, N) in enumerate(layers):
        if fmt == "int4":
            lay = synth.int4_layer(M, K, N, G, seed=rank, layer=li)
            qw = torch.from_numpy(lay.qweight).to(dev)
            sc = torch.from_numpy(lay.scales.view(np.int16)).to(dev)
            parts = FUSED_PARTS.get((args.workload, li))
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
            weights.append([packed] + [packed.clone() for _ in range(pool - 1)])
            wss.append(torch.zeros(mxg.w4a16_workspace_bytes(M, N, K, G), dtype=torch.uint8,
                                   device=dev))
        elif fmt == "int8":
            lay = synth.int8_layer(M, K, N, G, seed=rank, layer=li)
            qw = torch.from_numpy(lay.qweight).to(dev)
            sc = torch.from_numpy(lay.scales.view(np.int16)).to(dev)
            packed = mxg.w8a16_repack(qw, sc, G)
            del qw, sc
            weights.append([packed] + [packed.clone() for _ in range(pool - 1)])
            wss.append(torch.zeros(mxg.raw_lib().w8a16_workspace_bytes(M, N, K, G),
                                   dtype=torch.uint8, device=dev))
        elif fmt == "bf16":
            lay = synth.bf16_layer(M, K, N, seed=rank, layer=li)
            w = torch.from_numpy(lay.W.view(np.int16)).view(torch.bfloat16).to(dev)
            weights.append([w] + [w.clone() for _ in range(pool - 1)])
            wss.append(torch.zeros(mxg.raw_lib().bf16_gemm_small_workspace_bytes(M, N, K),
                                   dtype=torch.uint8, device=dev))
        else:
            lay = synth.mxfp8_layer(M, K, N, seed=rank, layer=li)
            wq = torch.from_numpy(lay.Wq).to(dev)
            ws = torch.from_numpy(lay.Ws).to(dev)
            weights.append([(wq, ws)] + [(wq.clone(), ws.clone()) for _ in range(pool - 1)])
            wss.append(torch.zeros(mxg.mxfp8_workspace_bytes(M, N, K), dtype=torch.uint8,
                                   device=dev))
        xs.append(torch.from_numpy(lay.X.view(np.int16)).view(torch.bfloat16).to(dev))
        ys.append(torch.empty((M, N), dtype=torch.bfloat16, device=dev))

    stream = torch.cuda.Stream(dev)

    def layer_call(li, p, s):
        K, N = layers[li]
        if fmt == "int4":
            mxg.w4a16_gemm(xs[li], weights[li][p], N, K, G, out=ys[li], workspace_buf=wss[li],
                           stream=s)
        elif fmt == "int8":
            mxg.w8a16_gemm(xs[li], weights[li][p], N, K, G, out=ys[li], workspace_buf=wss[li],
                           stream=s)
        elif fmt == "bf16":
            mxg.bf16_gemm_small(xs[li], weights[li][p], out=ys[li], workspace_buf=wss[li],
                                stream=s)
        else:
            wq, ws = weights[li][p]
            mxg.mxfp8_gemm(xs[li], wq, ws, out=ys[li], workspace_buf=wss[li], stream=s)

    # Graphs: a step is every layer once on pool slot p.  Plain graphs (one
    # per slot) time the steps; a second set with an event pair around every
    # launch times the kernels themselves (two sets, so one can be read while
    # the other runs).
    nl = len(layers)
    with torch.cuda.stream(stream):
        for li in range(nl):
            layer_call(li, 0, stream)           # plans and kernel attributes outside capture
        torch.cuda.synchronize(dev)
        graphs = []
        for p in range(pool):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for li in range(nl):
                    layer_call(li, p, stream)
            graphs.append(g)
    warmup, steps = args.warmup, args.steps
    with torch.cuda.stream(stream):          # replay() launches on the current stream
        for i in range(warmup):
            graphs[i % pool].replay()
    torch.cuda.synchronize(dev)
    status = max(abs(mxg.mxg_workspace_status(w)) for w in wss)
    if status:
        raise RuntimeError(f"kernel reported status {-status}")

    clocks = ClockSampler(local_rank)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t_start.record(stream)
        for i in range(steps):
            graphs[i % pool].replay()
        t_end.record(stream)
    torch.cuda.synchronize(dev)
    elapsed_ms = t_start.elapsed_time(t_end)

    # kernel durations over a second live pass: the stream is held by a
    # sleep kernel while a batch of launches, each between two events, is
    # queued behind it, so every event pair brackets exactly one kernel
    kernel_ms = [0.0] * nl
    kernel_launches = 0
    want = max(pool, min(steps, args.kernel_steps))
    batch = 64
    with torch.cuda.stream(stream):
        while kernel_launches < want:
            nb_steps = min(batch, want - kernel_launches)
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * nl * nb_steps)]
            torch.cuda._sleep(20_000_000)
            for i in range(nb_steps):
                p = (kernel_launches + i) % pool
                for li in range(nl):
                    evs[2 * (i * nl + li)].record(stream)
                    layer_call(li, p, stream)
                    evs[2 * (i * nl + li) + 1].record(stream)
            torch.cuda.synchronize(dev)
            for i in range(nb_steps):
                for li in range(nl):
                    kernel_ms[li] += evs[2 * (i * nl + li)].elapsed_time(evs[2 * (i * nl + li) + 1])
            kernel_launches += nb_steps
    if world > 1:
        dist.barrier()
    clk = clocks.stop()

    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    ms_per_step = elapsed_ms / steps

    # ------------------------------------------------------------- e2e arm
    e2e_steps = max(1, min(args.e2e_steps, steps))
    # one pinned host buffer holds every layer's X (and one every layer's Y):
    # a step copies X in once, runs the layers, and reads Y back once
    x_sizes = [x.numel() for x in xs]
    y_sizes = [y.numel() for y in ys]
    host_x = torch.cat([x.reshape(-1).cpu() for x in xs]).pin_memory()
    host_y = torch.empty(sum(y_sizes), dtype=torch.bfloat16).pin_memory()
    dev_xbuf = torch.empty(sum(x_sizes), dtype=torch.bfloat16, device=dev)
    dev_ybuf = torch.empty(sum(y_sizes), dtype=torch.bfloat16, device=dev)
    dev_x = [v.view(x.shape) for v, x in zip(torch.split(dev_xbuf, x_sizes), xs)]
    dev_y = [v.view(y.shape) for v, y in zip(torch.split(dev_ybuf, y_sizes), ys)]
    h2d = host_x.numel() * 2
    d2h = host_y.numel() * 2

    # the layer calls of every pool slot, marshalled once (binding.prepare_*)
    prepared = []
    for p in range(pool):
        calls = []
        for li, (K, N) in enumerate(layers):
            if fmt == "int4":
                c, _ = mxg.prepare_w4a16_gemm(dev_x[li], weights[li][p], N, K, G, out=dev_y[li],
                                              workspace_buf=wss[li], stream=stream)
            elif fmt == "int8":
                c, _ = mxg.prepare_w8a16_gemm(dev_x[li], weights[li][p], N, K, G, out=dev_y[li],
                                              workspace_buf=wss[li], stream=stream)
            elif fmt == "bf16":
                c, _ = mxg.prepare_bf16_gemm_small(dev_x[li], weights[li][p], out=dev_y[li],
                                                   workspace_buf=wss[li], stream=stream)
            else:
                wq, ws = weights[li][p]
                c, _ = mxg.prepare_mxfp8_gemm(dev_x[li], wq, ws, out=dev_y[li],
                                              workspace_buf=wss[li], stream=stream)
            calls.append(c)
        prepared.append(calls)

    def e2e_step(p):
        dev_xbuf.copy_(host_x, non_blocking=True)
        for call in prepared[p]:
            call()
        host_y.copy_(dev_ybuf, non_blocking=True)

    # A serving loop replays the step as a CUDA graph: one graph per pool slot
    # holding the step's host-to-device copy, its layer calls (the prepared
    # binding calls) and its device-to-host copy.
    with torch.cuda.stream(stream):
        for i in range(3):
            e2e_step(i % pool)
        torch.cuda.synchronize(dev)
        e2e_graphs = []
        for p in range(pool):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                e2e_step(p)
            e2e_graphs.append(g)
        for i in range(3):
            e2e_graphs[i % pool].replay()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_graphs[i % pool].replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    peaks, peak_kind = load_peaks()
    if tensor_bound:
        unit = "TFLOP/s"
        value = job_value(step_flops * steps, world, elapsed_ms) / 1e12
        e2e_value = job_value(step_flops * e2e_steps, world, e2e_ms) / 1e12
    else:
        unit = "TB/s"
        value = job_value(step_bytes * steps, world, elapsed_ms) / 1e12
        e2e_value = job_value(step_bytes * e2e_steps, world, e2e_ms) / 1e12

    # dominant kernel: every layer of the step runs the same kernel
    k_total_ms = sum(kernel_ms)
    if tensor_bound:
        achieved = step_flops * kernel_launches / (k_total_ms * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                "peak_source": f"{peak_kind} bf16 dense (burst)"}
    else:
        achieved = step_bytes * kernel_launches / (k_total_ms * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                "frac": round(achieved / peak, 4), "traffic": None,
                "peak_source": f"{peak_kind} copy bandwidth"}
    kernel_name = ("bf16_small_kernel" if fmt == "bf16" else
                   "w4a16_stream_kernel" if (fmt in ("int4", "int8") and M <= 32) else
                   "mxfp8_stream_kernel" if M <= 32 else "tc_gemm_kernel")
    roof["kernel"] = kernel_name
    roof["per_layer_us"] = [round(k / kernel_launches * 1e3, 3) for k in kernel_ms]
    roof["timed_launches"] = kernel_launches * nl
    traffic = traffic_from_profiles(kernel_name, args.workload)
    if traffic is not None:
        roof["traffic"] = traffic

    line = {
        "metric": "W4A16/MXFP8 GEMM weight-stream TB/s and TFLOP/s vs roofline, M=1..8192",
        "value": round(value, 4),
        "unit": unit,
        "n_gpus": world,
        "steps": steps,
        "warmup": warmup,
        "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",  # every path multiplies bf16 operands with fp32 accumulation
        "data": "synthetic (seeded; the value distributions of the layer formats)",
        "config": {
            "workload": args.workload,
            "format": fmt, "M": M, "layers_KxN": [f"{K}x{N}" for K, N in layers],
            "group_size": G if fmt in ("int4", "int8") else (32 if fmt == "mxfp8" else None),
            "weight_bytes_per_step": step_bytes, "flops_per_step": step_flops,
            "l2": f"rotating weight pool of {pool} copies ({pool * step_bytes / 1e6:.0f} MB >= "
                  f"{args.pool_factor:g} x L2)",
            "timing": "CUDA graphs of one step per pool slot, CUDA events on the launch stream; "
                      "kernel durations from a second live pass with an event pair around "
                      "each launch, queued behind a sleep kernel",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
        },
        "tflops": round(step_flops * steps / (elapsed_ms * 1e-3) / 1e12 * world, 3),
        "tbps": round(step_bytes * steps / (elapsed_ms * 1e-3) / 1e12 * world, 4),
        "e2e": {"value": round(e2e_value, 4), "unit": unit, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "path": "python binding (calls prepared once), the step captured once per "
                        "pool slot as a CUDA graph and replayed: per step one pinned-host copy "
                        "of every layer's X in, the layers, one copy of every layer's Y out"},
        "roofline": roof,
        "gpu_launches": len(layers) * steps,
        "clocks": clk,
        "gpu": props.name,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=args.cpu_budget)
    if world > 1:
        graphs.clear()
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


def cpu_baseline(workload: str, budget_s: float = 20.0):
    import oracle
    oracle.build()
    cores = os.cpu_count() or 1
    used = oracle.threads(cores)
    fmt, M, layers, G = WORKLOADS[workload]
    # size the column slice so one pass stays within the budget
    probe, _ = oracle_step_runner(workload, 64)
    t0 = time.perf_counter()
    b, f = probe(used)
    dt = max(time.perf_counter() - t0, 1e-6)
    full_cols = max(N for _, N in layers)
    cols = int(min(full_cols, max(64, 64 * budget_s / dt / 2)))
    run, _ = oracle_step_runner(workload, cols)
    t0 = time.perf_counter()
    b, f = run(used)
    dt = time.perf_counter() - t0
    # whole passes until about half the budget is spent (the first one counts)
    passes = 1
    while time.perf_counter() - t0 < 0.5 * budget_s:
        run(used)
        passes += 1
    dt = time.perf_counter() - t0
    b, f = b * passes, f * passes
    tensor_bound = workload in TENSOR_BOUND
    value = (f / dt / 1e12) if tensor_bound else (b / dt / 1e12)
    return {"value": value, "unit": "TFLOP/s" if tensor_bound else "TB/s", "cores": used,
            "kind": "oracle",
            "sample": f"{cols} of the output columns of every layer of {workload} "
                      f"(M={M}), {passes} pass(es), {dt:.1f} s, fp64 C oracle, "
                      f"OpenMP over columns"}


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
        "metric": "W4A16/MXFP8 GEMM weight-stream TB/s and TFLOP/s vs roofline, M=1..8192",
        "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; the value distributions of the layer formats)",
        "config": {"workload": args.workload, "format": fmt, "M": M,
                   "layers_KxN": [f"{K}x{N}" for K, N in layers]},
        "cpu_baseline": {"value": value, "unit": unit, "cores": used, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="mtp4_verify_int4")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--kernel-steps", type=int, default=512)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--ref-budget", type=float, default=120.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
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
