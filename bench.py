"""Benchmark: SVQ 2.25-bpw batch-1 GEMV on a Qwen3-4B-shaped decoder layer.

One step = one grouped launch of the seven SVQ linears of a decoder layer
(q 2560->4096 (6,4), k/v 2560->1024 (7,3)/(8,2), o 4096->2560 (9,1),
gate/up 2560->9728 (6,4)/(7,3), down 9728->2560 (8,2)) at batch 1, x fp16.
Steps rotate through 14 independent layer copies (397 MB of packed codes, more
than 3x the 126 MB L2), so every step streams its weights from HBM.  Launches
are replayed from CUDA graphs; the timed region is bracketed by a barrier and
device synchronisation and timed with CUDA events on the launching stream.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU: one process per GPU (torchrun); the layer is not partitioned, each
rank runs the same workload on its own GPU (replicas, weak scaling); the
reported value is the sum of all ranks' bytes over the slowest rank's time.
--impl reference: the CPU oracle on the host cores, same metric, each step a
bounded sample (8 rows of one of the seven matrices).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "SVQ 2.25-bpw GEMV packed-weight GB/s and % HBM peak (batch 1, Qwen3-4B shapes)"
UNIT = "GB/s"
N_LAYERS = 14
WORKLOAD = "qwen3-4b decoder layer: 7 SVQ linears (q,k,v,o,gate,up,down), batch 1, one grouped launch per step"


# DRAM bytes (read + written) of one GEMV launch on this workload, from an ncu
# capture of the kernel built from the sources whose hash is recorded here;
# reported only while the sources still hash to that value.
GEMV_TRAFFIC_CAPTURE = {
    "bytes": 28755712,
    "sources": ["gemv_impl.cuh", "gemv_device.cuh", "gemv.cu", "gemv_params.h", "gemv_mt1.cu", "layout.cuh",
                "svq_internal.h"],
    "sha256": "b30653bcb7ab36363a0568ee433dff2e0bd89eaafef293fd50d246f7f7f617a8",
}


def gemv_traffic():
    """Captured DRAM bytes per launch, or None once the kernel sources changed."""
    import hashlib
    h = hashlib.sha256()
    src = os.path.join(os.path.dirname(os.path.abspath(__file__)), "bit_spherical_vector_b200", "csrc")
    try:
        for f in GEMV_TRAFFIC_CAPTURE["sources"]:
            with open(os.path.join(src, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return GEMV_TRAFFIC_CAPTURE["bytes"] if h.hexdigest() == GEMV_TRAFFIC_CAPTURE["sha256"] else None


def layer_bytes():
    packed = sum(N * K * 9 // 32 for _, N, K in synth.QWEN3_4B_SHAPES)
    cb = sum((1 << b) * 16 for b in synth.QWEN3_4B_SPLITS)
    params = sum(N * 4 for _, N, K in synth.QWEN3_4B_SHAPES)          # fp16 scale + offset
    perm = sum(K * 4 for _, N, K in synth.QWEN3_4B_SHAPES)
    x = sum(K * 2 for _, N, K in synth.QWEN3_4B_SHAPES)
    y = sum(N * 4 for _, N, K in synth.QWEN3_4B_SHAPES)                # fp32 outputs
    return packed, packed + cb + params + perm + x + y


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [v.strip() for v in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def dist_init(backend: str | None = None):
    """One process per GPU, ranks from the launcher's environment.  NCCL on GPUs;
    `backend="gloo"` (or SVQ_BENCH_BACKEND=gloo) runs the same rank logic on CPUs."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        backend = backend or os.environ.get("SVQ_BENCH_BACKEND", "nccl")
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: float, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time (units/s)."""
    return world * units_per_rank / (ms_max * 1e-3)


# --------------------------------------------------------------------------- CPU oracle (reference arm, cpu_baseline)
def oracle_rows_sample(layer, step: int, rows: int = 8):
    """(bytes, seconds) of the oracle on `rows` rows of one matrix (chosen by `step`)."""
    import oracle
    m, x = layer[step % 7]
    nblk = m.N // rows
    r0 = ((step // 7) % nblk) * rows
    sub = synth.SvqMatrix(rows, m.K, m.b_d, np.ascontiguousarray(m.canonical[r0:r0 + rows]), m.codebook,
                          np.ascontiguousarray(m.scale[r0:r0 + rows]),
                          np.ascontiguousarray(m.offset[r0:r0 + rows]), m.perm)
    t0 = time.perf_counter()
    oracle.linear(sub, x)
    dt = time.perf_counter() - t0
    return rows * m.K * 9 // 32, dt


def _time_oracle(layer, budget_s: float):
    """The oracle on whole matrices of the layer (q, k, v, ... in turn) until budget_s has elapsed."""
    import oracle
    nbytes, secs, calls = 0, 0.0, 0
    while secs < budget_s:
        m, x = layer[calls % 7]
        t0 = time.perf_counter()
        oracle.linear(m, x)
        secs += time.perf_counter() - t0
        nbytes += m.N * m.K * 9 // 32
        calls += 1
    return nbytes, secs, calls


def cpu_baseline(layer, budget_s: float = 12.0, single_budget_s: float = 8.0):
    """The oracle on all host threads (OpenMP over rows) and, beside it, on one thread."""
    import oracle
    oracle.linear(*layer[1])  # warm (builds the library)
    cores = oracle.num_threads()
    nbytes, secs, calls = _time_oracle(layer, budget_s)
    oracle.set_threads(1)
    try:
        nb1, secs1, calls1 = _time_oracle(layer, single_budget_s)
    finally:
        oracle.set_threads(cores)
    return {"value": nbytes / secs / 1e9, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{calls} calls of the fp64 C++ oracle, each one whole matrix of the layer in turn "
                      f"(q, k, v, o, gate, up, down: decode + fp64 dot), {nbytes} packed bytes in {secs:.1f} s",
            "single_thread": {"value": nb1 / secs1 / 1e9, "unit": UNIT, "cores": 1,
                              "sample": f"{calls1} whole-matrix calls, {nb1} packed bytes in {secs1:.1f} s"}}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    layer = synth.qwen3_4b_layer(0)
    import oracle
    oracle.linear(*layer[1])
    for s in range(args.warmup):
        oracle_rows_sample(layer, s)
    nbytes, secs = 0, 0.0
    t_end = time.perf_counter() + 150.0            # the whole run ends within a few minutes
    done = 0
    for s in range(args.steps):
        b, dt = oracle_rows_sample(layer, args.warmup + s)
        nbytes += b
        secs += dt
        done += 1
        if time.perf_counter() > t_end:
            break
    value = nbytes / secs / 1e9
    cores = oracle.num_threads()
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs / done * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference", "steps_done": done,
            "config": {"workload": WORKLOAD + " (CPU oracle: 8-row sample of one matrix per step)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "8 rows of one of the seven matrices per step, fp64 C++ oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- GPU arm
def run_gpu(args, world, rank, local):
    import torch

    import bit_spherical_vector_b200 as svq

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    packed_b, alg_b = layer_bytes()

    # Weights: N_LAYERS independent layer copies resident in HBM.
    layers, Ws, xs_host = [], [], []
    with torch.cuda.stream(stream):
        for L in range(N_LAYERS):
            layer = synth.qwen3_4b_layer(L)
            layers.append(layer)
            Ws.append([svq.SvqWeight.from_synth(m) for m, _ in layer])
            xs_host.append([x for _, x in layer])
    torch.cuda.synchronize()
    for W in Ws:                      # drop the canonical upload buffers
        for w in W:
            w._canon_d = None

    # One contiguous device buffer per layer for the seven inputs and one for the
    # seven outputs (views per matrix), so the end-to-end leg moves each step's
    # activations with one copy each way.
    y_len = [sum(m.N for m, _ in layer) for layer in layers]
    xbuf = [torch.from_numpy(np.concatenate([x.reshape(-1) for x in xl]).view(np.int16)).to(dev).view(torch.float16)
            for xl in xs_host]
    ybuf = [torch.empty(n, dtype=torch.float32, device=dev) for n in y_len]

    def views(buf, sizes, shapes):
        out, o = [], 0
        for n, shp in zip(sizes, shapes):
            out.append(buf[o:o + n].view(shp))
            o += n
        return out

    xs = [views(xbuf[L], [x.size for x in xs_host[L]], [x.shape for x in xs_host[L]]) for L in range(N_LAYERS)]
    ys = [views(ybuf[L], [m.N for m, _ in layers[L]], [(1, m.N) for m, _ in layers[L]]) for L in range(N_LAYERS)]
    nb = max(svq.svq_linear_gemv_batched_workspace_size(W, 1) for W in Ws)
    ws = torch.empty(max(nb, 256), dtype=torch.uint8, device=dev)
    with torch.cuda.stream(stream):
        svq.svq_workspace_init(ws)

    def step(i):
        L = i % N_LAYERS
        svq.svq_linear_gemv_batched(Ws[L], xs[L], ys[L], ws)

    # warm-up (eager), then capture one graph per layer and one graph of all layers
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            step(i)
    torch.cuda.synchronize()
    g_all = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_all, stream=stream):
        for i in range(N_LAYERS):
            step(i)
    g_one = []
    for L in range(N_LAYERS):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(L)
        g_one.append(g)

    def replay(k):
        full, rem = divmod(k, N_LAYERS)
        for _ in range(full):
            g_all.replay()
        for L in range(rem):
            g_one[L].replay()

    with torch.cuda.stream(stream):
        replay(N_LAYERS * 4)          # graph warm-up
    torch.cuda.synchronize()

    # ---- device-timed region: K steps per region, regions repeated until at least
    # 200 ms have been timed (clocks sampled throughout); the median region gives
    # the per-step time (each region is bracketed by barrier + synchronize and
    # timed with CUDA events on the launching stream, max over ranks)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed_region():
        barrier(world)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ev0.record(stream)
            replay(args.steps)
            ev1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        return max_over_ranks(ev0.elapsed_time(ev1), world)

    region_ms = []
    with ClockSampler(local) as clk:
        region_ms.append(timed_region())
        repeats = min(200, max(1, int(np.ceil(200.0 / max(region_ms[0], 1e-3)))))
        # every rank takes the same number of steps (rank 0's count is broadcast)
        repeats = int(max_over_ranks(float(repeats), world))
        for _ in range(repeats - 1):
            region_ms.append(timed_region())
    ms_max = float(np.median(region_ms))
    value = job_rate(world, args.steps * packed_b, ms_max) / 1e9
    per_launch_s = ms_max * 1e-3 / args.steps
    peak, peak_kind = read_peaks()
    achieved = alg_b / per_launch_s / 1e9

    # ---- end-to-end through the public API, one step at a time: one
    # svq_linear_gemv_batched_host call through the C ABI per step, which copies
    # the step's inputs from pinned host memory, runs the layer and copies the
    # outputs back to pinned host memory, all in order on one stream (nothing of
    # one step overlaps the next)
    e2e_steps = min(args.steps, 2000)
    xh = [xb.cpu().pin_memory() for xb in xbuf]
    yh = [torch.empty(n, dtype=torch.float32).pin_memory() for n in y_len]
    h2d = xh[0].numel() * 2
    d2h = yh[0].numel() * 4
    calls = [svq.GemvBatchCall(Ws[L], xs[L], ys[L], ws) for L in range(N_LAYERS)]
    host_calls = [svq.GemvBatchHostCall(Ws[L], 1, xh[L], xbuf[L], yh[L], ybuf[L], ws) for L in range(N_LAYERS)]

    def e2e_step(i):
        host_calls[i % N_LAYERS](stream)

    with torch.cuda.stream(stream):
        for i in range(2 * N_LAYERS):
            e2e_step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = job_rate(world, e2e_steps * packed_b, e2e_ms) / 1e9

    # ---- the same, as a deployment would run it: one CUDA graph per N_LAYERS steps,
    # the copies on their own streams chained by events, so one step's copies
    # overlap the next step's layer
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=stream):
        fork = torch.cuda.Event()
        fork.record(stream)
        h2d_s.wait_event(fork)
        d2h_s.wait_event(fork)
        ev_in = [torch.cuda.Event() for _ in range(N_LAYERS)]
        ev_k = [torch.cuda.Event() for _ in range(N_LAYERS)]
        ev_out = [torch.cuda.Event() for _ in range(N_LAYERS)]
        for L in range(N_LAYERS):
            with torch.cuda.stream(h2d_s):
                xbuf[L].copy_(xh[L], non_blocking=True)
                ev_in[L].record(h2d_s)
            stream.wait_event(ev_in[L])
            calls[L](stream)
            ev_k[L].record(stream)
            d2h_s.wait_event(ev_k[L])
            with torch.cuda.stream(d2h_s):
                yh[L].copy_(ybuf[L], non_blocking=True)
                ev_out[L].record(d2h_s)
        stream.wait_event(ev_in[N_LAYERS - 1])
        stream.wait_event(ev_out[N_LAYERS - 1])
    replays = (e2e_steps + N_LAYERS - 1) // N_LAYERS
    eg_steps = replays * N_LAYERS
    with torch.cuda.stream(stream):
        g_e2e.replay()                                   # warm-up
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(replays):
            g_e2e.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    eg_ms = max_over_ranks(e0.elapsed_time(e1), world)
    eg_value = job_rate(world, eg_steps * packed_b, eg_ms) / 1e9
    del g_e2e

    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layer_packed_bytes": packed_b, "layer_algorithmic_bytes": alg_b,
                   "layer_copies_rotated": N_LAYERS,
                   "l2": f"inputs larger than L2: {N_LAYERS} layer copies, {N_LAYERS * packed_b / 1e6:.0f} MB "
                         "of packed codes rotated",
                   "hbm_pct_of_peak": 100.0 * value / world / peak, "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": gemv_traffic(),
                     "peak_source": f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)" if peak_kind == "measured"
                     else "fallback 6650 GB/s",
                     "kernel": "gemv_kernel<1, 1> (grouped, 7 matrices)",
                     "achieved_bytes": "all algorithmic bytes per launch (packed codes, codebooks, radius "
                                       "params, perm, x, y)"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps,
                "how": "every step in order on one stream: one svq_linear_gemv_batched_host call through "
                       "the C ABI (pinned host x -> device copy, the grouped launch, device -> pinned host "
                       "y copy)"},
        "e2e_graph": {"value": eg_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                      "steps": eg_steps,
                      "how": f"the same steps captured {N_LAYERS} per CUDA graph, copies on their own streams "
                             "chained by events so one step's copies overlap the next step's layer"},
        "timing": {"regions": len(region_ms), "steps_per_region": args.steps,
                   "region_ms_median": ms_max, "region_ms_min": min(region_ms), "region_ms_max": max(region_ms),
                   "timed_ms_total": float(sum(region_ms))},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(layers[0])
    if world == 1 and not args.no_secondary:
        del g_all, g_one
        line["secondary"] = {"sweep_8192": run_sweep(args, quiet=True), "prefill": run_prefill(args, quiet=True),
                             "moe": run_moe(args, quiet=True), "calibration": run_calib(args, quiet=True),
                             "layer_radius_tables": run_lut_layer(args, quiet=True),
                             "shape_tails": run_tails(args, quiet=True)}
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------- secondary workloads
def _time_graph(fn, reps, stream):
    """Capture fn() once in a CUDA graph, replay `reps` times; return microseconds per replay."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) * 1e3 / reps


def run_sweep(args, quiet=False):
    """8192 x 8192 (7,3) matrix, M = 1..16 tokens: GEMV and tensor-core GEMM, 20 rotated copies (378 MB)."""
    recs = []
    import torch
    import bit_spherical_vector_b200 as svq
    stream = torch.cuda.Stream()
    copies = 20
    base = synth.square_8192()
    Ws = []
    for c in range(copies):
        m = synth.make_matrix(2, 100 + c, 8192, 8192, 7) if c else base
        Ws.append(svq.SvqWeight.from_synth(m))
    torch.cuda.synchronize()
    packed = 8192 * 8192 * 9 // 32
    for M in (1, 2, 4, 8, 16):
        x = torch.from_numpy(synth.square_8192_x(M).view(np.int16)).cuda().view(torch.float16)
        y = torch.empty((M, 8192), dtype=torch.float32, device="cuda")
        nbv = svq.svq_linear_gemv_workspace_size(Ws[0], M)
        wsv = torch.empty(max(nbv, 256), dtype=torch.uint8, device="cuda")
        nbg = svq.svq_linear_gemm_workspace_size(Ws[0], M)
        wsg = torch.empty(max(nbg, 256), dtype=torch.uint8, device="cuda")
        with torch.cuda.stream(stream):
            svq.svq_workspace_init(wsv)
            svq.svq_workspace_init(wsg)

        def gemv():
            for W in Ws:
                svq.svq_linear_gemv(W, x, y, wsv)

        def gemm():
            for W in Ws:
                svq.svq_linear_gemm(W, x, y, wsg)
        tv = _time_graph(gemv, 20, stream) / copies
        tg = _time_graph(gemm, 20, stream) / copies
        rec = {"workload": "sweep 8192x8192 (7,3)", "M": M, "gemv_us": round(tv, 3),
               "gemv_GBps": round(packed / tv / 1e3, 1), "gemm_us": round(tg, 3),
               "gemm_GBps": round(packed / tg / 1e3, 1), "faster": "gemv" if tv <= tg else "gemm",
               "tokens_per_s_best": round(M / min(tv, tg) * 1e6, 1)}
        recs.append(rec)
        if not quiet:
            print(json.dumps(rec), flush=True)
    cross = next((r["M"] for r in recs if r["faster"] == "gemm"), None)
    if quiet:
        return {"per_M": recs, "gemv_to_gemm_crossover_M": cross}
    return 0


def run_prefill(args, quiet=False):
    """Qwen3-4B gate/up (2560->9728) and down (9728->2560), (8,2), M = 512 and 2048, bf16."""
    recs = []
    import torch
    import bit_spherical_vector_b200 as svq
    stream = torch.cuda.Stream()
    peak, kind = read_peaks()
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            tpeak = float(json.load(f)["bf16_tflops"])
    except Exception:
        tpeak = 1590.0
    for which, m in enumerate(synth.prefill_mats()):
        W = svq.SvqWeight.from_synth(m)
        wq = torch.empty((m.N, m.K), dtype=torch.bfloat16, device="cuda")
        svq.svq_dequantize(W, wq)
        for M in (512, 2048):
            x = torch.from_numpy(synth.prefill_x(M, m.K, which).view(np.int16)).cuda().view(torch.bfloat16)
            y = torch.empty((M, m.N), dtype=torch.float32, device="cuda")
            nb = svq.svq_linear_gemm_workspace_size(W, M)
            ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
            with torch.cuda.stream(stream):
                svq.svq_workspace_init(ws)
            t = _time_graph(lambda: svq.svq_linear_gemm(W, x, y, ws), 20, stream)
            xp = x[:, torch.from_numpy(m.perm.astype(np.int64)).cuda()].contiguous()
            yc = torch.empty((M, m.N), dtype=torch.bfloat16, device="cuda")
            tc = _time_graph(lambda: torch.matmul(xp, wq.t(), out=yc), 20, stream)
            flop = 2.0 * M * m.N * m.K
            rec = {"workload": f"prefill {m.K}->{m.N} (8,2) bf16", "M": M, "svq_gemm_us": round(t, 2),
                   "svq_TFLOPs": round(flop / t / 1e6, 1),
                   "svq_frac_of_bf16_peak": round(flop / t / 1e6 / tpeak, 3),
                   "cublas_dense_bf16_us": round(tc, 2), "cublas_TFLOPs": round(flop / tc / 1e6, 1),
                   "peak_bf16_TFLOPs": tpeak, "note": "svq time includes the x[:,perm] pass"}
            recs.append(rec)
            if not quiet:
                print(json.dumps(rec), flush=True)
    return recs if quiet else 0


def run_moe(args, quiet=False):
    """Qwen3-30B-A3B-shaped MoE FFN (hidden 2048, 128 experts, inter 768, top-8), T = 1 and 16."""
    recs = []
    import torch
    import bit_spherical_vector_b200 as svq
    stream = torch.cuda.Stream()
    experts = synth.moe_experts()
    gu, down = [], []
    for g, u, d in experts:
        gu += [svq.SvqWeight.from_synth(g), svq.SvqWeight.from_synth(u)]
        down.append(svq.SvqWeight.from_synth(d))
    gu_tab, dn_tab = svq.descriptor_table(gu), svq.descriptor_table(down)
    per_mat = 768 * 2048 * 9 // 32
    for T in (1, 16):
        ids, w = synth.moe_routing(T)
        k = ids.shape[1]
        e = torch.from_numpy(ids.astype(np.int64)).cuda().reshape(-1)
        tok = torch.arange(T, device="cuda").repeat_interleave(k)
        pair = torch.arange(T * k, device="cuda")
        items1 = svq.item_table(torch.stack([2 * e, 2 * e + 1], 1).reshape(-1), tok.repeat_interleave(2),
                                torch.stack([2 * pair, 2 * pair + 1], 1).reshape(-1), torch.ones(2 * T * k, device="cuda"))
        items2 = svq.item_table(e, pair, tok, torch.from_numpy(w.reshape(-1)).cuda())
        x = torch.from_numpy(synth.moe_x(T).view(np.int16)).cuda().view(torch.float16)
        y1 = torch.empty((2 * T * k, 768), dtype=torch.float32, device="cuda")
        out = torch.empty((T, 2048), dtype=torch.float32, device="cuda")
        ws1 = torch.empty(svq.svq_moe_grouped_gemv_workspace_size(len(gu), 2 * T * k, 768, False), dtype=torch.uint8,
                          device="cuda")
        ws2 = torch.empty(svq.svq_moe_grouped_gemv_workspace_size(len(down), T * k, 2048, True), dtype=torch.uint8,
                          device="cuda")

        def ffn():
            svq.svq_moe_grouped_gemv(gu_tab, len(gu), 768, 2048, 8, items1, 2 * T * k, T, x, svq.SVQ_X_F16, y1,
                                     2 * T * k, False, ws1)
            svq.svq_moe_grouped_gemv(dn_tab, len(down), 2048, 768, 8, items2, T * k, T, y1.view(T * k, 1536),
                                     svq.SVQ_X_SWIGLU_F32, out, T, True, ws2)
        t = _time_graph(ffn, 50, stream)
        touched = len(set(ids.reshape(-1).tolist()))
        nbytes = touched * 3 * per_mat
        rec = {"workload": "moe ffn qwen3-30b-a3b shapes", "T": T, "us": round(t, 2),
               "tokens_per_s": round(T / t * 1e6, 1), "experts_touched": touched,
               "GBps_distinct_packed": round(nbytes / t / 1e3, 1),
               "note": "L2-warm: the same routed experts every replay"}
        recs.append(rec)
        if not quiet:
            print(json.dumps(rec), flush=True)
    return recs if quiet else 0


def run_lut_layer(args, quiet=False):
    """The headline decoder layer (one grouped launch, batch 1, 14 rotated copies) with every matrix
    carrying a per-row radius table (2^b_r fp16 levels) instead of the affine scale/offset."""
    import torch
    import bit_spherical_vector_b200 as svq
    stream = torch.cuda.Stream()
    layers = []
    for L in range(N_LAYERS):
        mats = []
        for i, (m, x) in enumerate(synth.qwen3_4b_layer(L)):
            m.lut = synth.make_lut(500 + L, i, m.N, m.b_d)
            mats.append((svq.SvqWeight.from_synth(m),
                         torch.from_numpy(x.view(np.int16)).cuda().view(torch.float16)))
        layers.append(mats)
    ys = [[torch.empty((1, W.N), dtype=torch.float32, device="cuda") for W, _ in mats] for mats in layers]
    Ws0 = [W for W, _ in layers[0]]
    ws = torch.zeros(max(svq.svq_linear_gemv_batched_workspace_size(Ws0, 1), 256), dtype=torch.uint8, device="cuda")
    calls = [svq.GemvBatchCall([W for W, _ in mats], [x for _, x in mats], y, ws) for mats, y in zip(layers, ys)]

    def chain():
        for c in calls:
            c()
    us = _time_graph(chain, 50, stream) / N_LAYERS
    packed = sum(N * K * 9 // 32 for _, N, K in synth.QWEN3_4B_SHAPES)
    tables = sum(N * 2 * (1 << (10 - b)) for (_, N, K), b in zip(synth.QWEN3_4B_SHAPES, synth.QWEN3_4B_SPLITS))
    rec = {"workload": "qwen3-4b decoder layer, batch 1, per-row radius tables", "us_per_layer": round(us, 3),
           "GBps_packed": round(packed / us / 1e3, 1), "table_bytes_per_layer": tables}
    if not quiet:
        print(json.dumps(rec), flush=True)
    return [rec] if quiet else 0


def run_tails(args, quiet=False):
    """Shape tails: the batch-1 GEMV on a gate-shaped matrix whose N is not a multiple of 4 and whose K is
    not a multiple of 128 (9726 x 2552, stored padded to 9728 x 2560 with zero codes), against the aligned
    9728 x 2560; (8,2), 14 rotated copies each (larger than L2), one launch per copy."""
    import torch
    import bit_spherical_vector_b200 as svq
    stream = torch.cuda.Stream()
    recs = []
    for N, K in ((9728, 2560), (9726, 2552)):
        Ws, xs, ys = [], [], []
        for L in range(N_LAYERS):
            Ws.append(svq.SvqWeight.from_synth(synth.make_matrix(600 + L, 0, N, K, 8)))
            xs.append(torch.from_numpy(synth.make_x(600 + L, 1, 1, K).view(np.int16)).cuda().view(torch.float16))
            ys.append(torch.empty((1, N), dtype=torch.float32, device="cuda"))
        ws = torch.zeros(max(svq.svq_linear_gemv_workspace_size(Ws[0], 1), 256), dtype=torch.uint8, device="cuda")
        calls = [svq.GemvBatchCall([W], [x], [y], ws) for W, x, y in zip(Ws, xs, ys)]

        def chain():
            for c in calls:
                c()
        us = _time_graph(chain, 50, stream) / N_LAYERS
        stored = svq.svq_packed_bytes(N, K)
        recs.append({"workload": f"gemv {N}x{K} (8,2), batch 1", "us": round(us, 3),
                     "packed_bytes_stored": stored, "packed_bytes_of_the_matrix": N * K * 9 // 32,
                     "GBps_stored": round(stored / us / 1e3, 1)})
        if not quiet:
            print(json.dumps(recs[-1]), flush=True)
    return recs if quiet else 0


def run_calib(args, quiet=False):
    """Calibration side on one gate-projection-shaped matrix (9728 x 2560): ESG from 512 calibration rows,
    then for each candidate split b_d 6..9 the radius grid and the activation-weighted encode, then ABS.
    Each step timed with CUDA events (median of 3)."""
    import torch
    import bit_spherical_vector_b200 as svq
    N, K, T = 9728, 2560, 512
    rng = np.random.default_rng(7)
    W = torch.from_numpy((rng.standard_normal((N, K)) * 0.02).astype(np.float32)).cuda()
    x = torch.from_numpy((rng.standard_normal((T, K)) * rng.lognormal(0.0, 1.0, K)[None, :]).astype(np.float32)).cuda()
    energy = torch.empty(K, dtype=torch.float64, device="cuda")
    perm = torch.empty(K, dtype=torch.int32, device="cuda")
    wts = torch.empty(K, dtype=torch.float32, device="cuda")
    splits = (6, 7, 8, 9)
    cbs = [torch.from_numpy(synth.make_codebook(synth.rng(7, b, synth.F_CODEBOOK), b).view(np.int16)).cuda()
           for b in splits]
    sc = [torch.empty(N, dtype=torch.int16, device="cuda") for _ in splits]
    of = [torch.empty(N, dtype=torch.int16, device="cuda") for _ in splits]
    canon = [torch.empty((N, synth.canonical_row_bytes(K)), dtype=torch.uint8, device="cuda") for _ in splits]
    row_err = torch.empty((len(splits), N), dtype=torch.float64, device="cuda")
    totals = torch.empty(len(splits), dtype=torch.float64, device="cuda")
    best = torch.empty(1, dtype=torch.int32, device="cuda")

    def timed(fn, reps=3):
        fn()
        torch.cuda.synchronize()
        out = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            out.append(e0.elapsed_time(e1) * 1e3)
        return float(np.median(out))

    rec = {"workload": "calibration 9728x2560 (gate shape), 512 calibration rows, splits b_d 6..9",
           "esg_us": round(timed(lambda: svq.svq_esg(x, 0.5, energy, perm, wts)), 1), "splits": []}
    nsub = N * K // 8
    for i, b in enumerate(splits):
        g_us = timed(lambda: svq.svq_radius_grid(W, perm, b, sc[i], of[i]))
        e_us = timed(lambda: svq.svq_encode(W, b, perm, wts, cbs[i], sc[i], of[i], canon[i], row_err[i]))
        rec["splits"].append({"b_d": b, "radius_grid_us": round(g_us, 1), "encode_us": round(e_us, 1),
                              "encode_Msubvectors_per_s": round(nsub / e_us, 1)})
    rec["abs_select_us"] = round(timed(lambda: svq.svq_abs_select(row_err, totals, best)), 1)
    rec["abs_choice_b_d"] = splits[int(best.item())]
    rec["total_ms"] = round((rec["esg_us"] + sum(d["radius_grid_us"] + d["encode_us"] for d in rec["splits"])
                             + rec["abs_select_us"]) / 1e3, 2)
    if not quiet:
        print(json.dumps(rec), flush=True)
    return [rec] if quiet else 0


def run_chain(args):
    """Qwen3-4B decoder-layer chain at batch 1 and 4: the layer's linears in dependency order with their
    producers (norm -> q|k|v, o, norm -> gate|up, SiLU-gated product -> down; attention itself is not part of
    the chain, o reads a synthetic attention output).  Two variants: the producers write x in natural order
    and every SVQ call gathers x[perm] ("gather"), or the producers write each consumer's stored order and the
    SVQ calls take perm NULL ("stored").  14 rotated layer copies (inputs larger than L2)."""
    import torch
    import bit_spherical_vector_b200 as svq
    stream = torch.cuda.Stream()
    packed_b, _ = layer_bytes()
    eps = float(np.float32(1e-6))
    layers = []
    for L in range(N_LAYERS):
        Ws = [svq.SvqWeight.from_synth(m) for m, _ in synth.qwen3_4b_layer(L)]
        layers.append((Ws, [W.without_perm() for W in Ws]))
    torch.cuda.synchronize()
    rng = np.random.default_rng(12)
    f16 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float16)).cuda()
    g1, g2 = f16(rng.uniform(0.5, 1.5, 2560)), f16(rng.uniform(0.5, 1.5, 2560))
    for M in (1, 4):
        h1 = torch.from_numpy(synth.make_x(12, 0, M, 2560, energies=True).view(np.int16)).cuda().view(torch.float16)
        h2 = torch.from_numpy(synth.make_x(12, 1, M, 2560, energies=True).view(np.int16)).cuda().view(torch.float16)
        att = torch.from_numpy(synth.make_x(12, 2, M, 4096).view(np.int16)).cuda().view(torch.float16)
        e16 = lambda k: torch.empty((M, k), dtype=torch.float16, device="cuda")
        xn, xn2, xd = e16(2560), e16(2560), e16(9728)
        xq, xk, xv, xg, xu = e16(2560), e16(2560), e16(2560), e16(2560), e16(2560)
        ys = [torch.empty((M, N), dtype=torch.float32, device="cuda") for _, N, _ in synth.QWEN3_4B_SHAPES]
        groups = lambda Ws: [Ws, Ws[0:3], Ws[3:4], Ws[4:6], Ws[6:7]]
        nb = max(svq.svq_linear_gemv_batched_workspace_size(G, M) for Ws, _ in layers for G in groups(Ws))
        ws = torch.empty(max(nb, 256), dtype=torch.uint8, device="cuda")
        with torch.cuda.stream(stream):
            svq.svq_workspace_init(ws)

        def gather():
            for Ws, _ in layers:
                svq.svq_rmsnorm_permute(h1, g1, eps, [None], [xn])
                svq.svq_linear_gemv_batched(Ws[0:3], [xn] * 3, ys[0:3], ws)
                svq.svq_linear_gemv(Ws[3], att, ys[3], ws)
                svq.svq_rmsnorm_permute(h2, g2, eps, [None], [xn2])
                svq.svq_linear_gemv_batched(Ws[4:6], [xn2] * 2, ys[4:6], ws)
                svq.svq_swiglu_permute(ys[4], ys[5], None, xd)
                svq.svq_linear_gemv(Ws[6], xd, ys[6], ws)

        def stored():
            for Ws, Wn in layers:
                svq.svq_rmsnorm_permute(h1, g1, eps, [W.perm for W in Ws[0:3]], [xq, xk, xv])
                svq.svq_linear_gemv_batched(Wn[0:3], [xq, xk, xv], ys[0:3], ws)
                svq.svq_linear_gemv(Ws[3], att, ys[3], ws)
                svq.svq_rmsnorm_permute(h2, g2, eps, [W.perm for W in Ws[4:6]], [xg, xu])
                svq.svq_linear_gemv_batched(Wn[4:6], [xg, xu], ys[4:6], ws)
                svq.svq_swiglu_permute(ys[4], ys[5], Ws[6].perm, xd)
                svq.svq_linear_gemv(Wn[6], xd, ys[6], ws)

        def stored_o():
            # as stored, with the attention output also taken in o's stored order
            for Ws, Wn in layers:
                svq.svq_rmsnorm_permute(h1, g1, eps, [W.perm for W in Ws[0:3]], [xq, xk, xv])
                svq.svq_linear_gemv_batched(Wn[0:3], [xq, xk, xv], ys[0:3], ws)
                svq.svq_linear_gemv(Wn[3], att, ys[3], ws)
                svq.svq_rmsnorm_permute(h2, g2, eps, [W.perm for W in Ws[4:6]], [xg, xu])
                svq.svq_linear_gemv_batched(Wn[4:6], [xg, xu], ys[4:6], ws)
                svq.svq_swiglu_permute(ys[4], ys[5], Ws[6].perm, xd)
                svq.svq_linear_gemv(Wn[6], xd, ys[6], ws)

        def one_launch():
            for Ws, _ in layers:
                svq.svq_linear_gemv_batched(Ws, [xn] * 3 + [att, xn2, xn2, xd], ys, ws)

        res = {}
        for name, fn in (("one_launch", one_launch), ("gather", gather), ("stored", stored), ("stored_o", stored_o)):
            res[name] = _time_graph(fn, 50, stream) / N_LAYERS
        print(json.dumps({"workload": "qwen3-4b decoder-layer chain", "M": M,
                          "us_per_layer": {k: round(v, 2) for k, v in res.items()},
                          "GBps_packed": {k: round(packed_b / v / 1e3, 1) for k, v in res.items()},
                          "launches_per_layer": {"one_launch": 1, "gather": 7, "stored": 7, "stored_o": 7},
                          "note": "one_launch = the seven linears in one grouped launch without their data "
                                  "dependencies (the headline); gather/stored = dependency order with producers; "
                                  "stored_o = stored with the attention output also in o's stored order"}),
              flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=140000)
    ap.add_argument("--warmup", type=int, default=1400)
    ap.add_argument("--impl", default="svq", choices=["svq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the sweep / prefill / MoE / calibration measurements added to the headline line")
    ap.add_argument("--workload", default="layer",
                    choices=["layer", "sweep", "prefill", "moe", "chain", "calib", "lut", "tails"],
                    help="layer = the headline line; the others print one JSON line per configuration")
    args = ap.parse_args()
    if args.workload != "layer":
        return {"sweep": run_sweep, "prefill": run_prefill, "moe": run_moe, "chain": run_chain,
                "calib": run_calib, "lut": run_lut_layer, "tails": run_tails}[args.workload](args)
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_init() if args.impl == "svq" else (int(os.environ.get("WORLD_SIZE", "1")),
                                                                 int(os.environ.get("RANK", "0")), 0)
    try:
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_gpu(args, world, rank, local)
    finally:
        if world > 1 and args.impl == "svq":
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
