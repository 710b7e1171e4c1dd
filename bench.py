"""Benchmark: fused W4A16 decode GEMV, HBM GB/s at M=1, K=4096, N=14336.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl wq|reference]

One step = one fused dequant-in-register matmul Y[1, 14336] = X[1, 4096] *
What^T over a Llama-8B gate/up-shaped INT4 layer (asymmetric, group 128,
binary16 scale and zero), inputs resident in HBM.  Successive steps read
different copies of the quantized layer from a pool larger than 4x the L2,
so every step streams its weights from HBM.  Steps are replayed from CUDA
graphs and timed with CUDA events on the launching stream.

value       = algorithmic bytes of all steps on all GPUs / device time (GB/s)
roofline    = the same per launch against the measured HBM copy bandwidth
e2e         = the same metric through the Python API with X on the host
              (pinned), copied in, and Y read back to the host every step
cpu_baseline= the CPU oracle (plain C, float64) on the same layer

For N > 1 (torchrun) each rank runs an independent replica on its own GPU
(the decode GEMV has no exchange step); time is the max over ranks.
``--impl reference`` times the CPU oracle as the reference arm.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A16 fused GEMV HBM GB/s (fraction of B200 peak) at M=1, K=4096, N=14336"
M, K, N = 1, 4096, 14336
BITS, GROUP, SYM = 4, 128, False
WORKLOAD = ("decode GEMV, Llama-8B gate/up layer: M=1, K=4096, N=14336, INT4 asymmetric "
            "group 128, fp16 scale+zero, bf16 X, fp32 Y")
FALLBACK_HBM_GBS = 6650.0
GRAPH_MAX_LAUNCHES = 4096      # larger step counts replay graphs of one pool cycle
SLEEP_CYCLES = 2_000_000       # ~1 ms of device time ahead of the start event
PROFILE_SUMMARY = os.path.join(ROOT, "profiles", "gemv_w4a16_m1_k4096_n14336.json")
CSRC = os.path.join(ROOT, "w4a16_decode_matmul_b200", "csrc")
# What decides the timed kernel: its device code, the host plan and launch of
# it, and the matmul entry point that chooses it.
KERNEL_SOURCES = [os.path.join(CSRC, f)
                  for f in ("gemv_ks.cuh", "gemv_ld.cuh", "unpack.cuh", "common.cuh", "k_ks.cu")]
KERNEL_HOST_SECTIONS = [
    ("wq_status wq_matmul(const void* X, int64_t M,",
     "// ------------------------------------------------------ no-allocation entry"),
]
# Page 2 ("量化", llminference s08, section 换来了什么): its bandwidth-model
# estimate for an 8B model on an H100 (~3.35 TB/s), quoted as context only.
PAGE2_H100_CONTEXT = {
    "kind": "context from the pages (another GPU, a bytes / bandwidth model), not a target",
    "source": "page 2 '量化' (llminference s08), section 换来了什么: 8B model on an H100",
    "fp16_ms_per_token": 4.78, "int4_group32_ms_per_token": 1.25,
    "note": ("the 1.25 ms uses 4.19 GiB as if it were GB; with 8e9 x 4.5 / 8 = 4.5e9 bytes "
             "the same model gives 1.34 ms"),
}


def algorithmic_bytes(m: int = M, n: int = N, k: int = K, bits: int = BITS,
                      group: int = GROUP, sym: bool = SYM, y_bytes: int = 4) -> int:
    """Bytes the method must move per step: packed codes + scales (+ zeros)
    + X + Y (page 1 section 2: N_param * b / 8 + metadata)."""
    meta = n * (k // group) * 2 * (1 if sym else 2)
    return n * k * bits // 8 + meta + m * k * 2 + m * n * y_bytes


def kernel_source_hash() -> str:
    """Hash of the sources that decide the timed kernel (device headers, its
    plan and launch in k_ks.cu, and the kernel choice in wq.cu)."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(f, "rb").read())
    host = open(os.path.join(CSRC, "wq.cu"), encoding="utf-8").read()
    for start, end in KERNEL_HOST_SECTIONS:
        i = host.index(start)
        h.update(host[i:host.index(end, i)].encode("utf-8"))
    return h.hexdigest()[:16]


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------- ranks

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(value: float, device=None) -> float:
    """Max of a float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(bytes_per_step: int, steps: int, world: int, max_ms: float) -> float:
    """Aggregate throughput: every rank moves bytes_per_step per step."""
    return bytes_per_step * steps * world / (max_ms * 1e-3) / 1e9


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.file = None

    def __enter__(self):
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                r = [x.strip() for x in r]
                sm.append(float(r[1]))
                mx.append(float(r[2]))
                for name, flag in zip(names, r[5:9]):
                    if flag.lower() == "active":
                        reasons.add(name)
            except (ValueError, IndexError):
                continue
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        top = sorted(sm)[len(sm) // 4:]        # samples taken under load
        return {"sm_mhz": statistics.median(top), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU oracle

def oracle_threads() -> int:
    return len(os.sched_getaffinity(0))


_ORACLE_INPUTS = {}


def time_oracle(target_s: float, seed_w: int = 0, seed_x: int = 1, threads: int | None = None):
    """Time the oracle's matmul (decode from codes + float64 dot products) on
    the same layer for about target_s seconds, with `threads` OpenMP threads
    (all affinity cores by default).  Returns (GB/s, steps, s)."""
    import oracle
    import synth
    orc = oracle.get()
    key = (seed_w, seed_x)
    if key not in _ORACLE_INPUTS:
        W = synth.weight(N, K, seed=seed_w)
        X = synth.activation(M, K, seed=seed_x)
        _, codes, scales, zeros = orc.quantize(synth.half_bits(W), BITS, GROUP, SYM)
        _ORACLE_INPUTS[key] = (codes, scales, zeros, synth.bf16_bits(X))
    codes, scales, zeros, xb = _ORACLE_INPUTS[key]
    orc.set_threads(threads or oracle_threads())
    steps, t0 = 0, time.perf_counter()
    while True:
        orc.matmul(xb, codes, scales, zeros, N, K, BITS, GROUP, SYM)
        steps += 1
        el = time.perf_counter() - t0
        if el >= target_s:
            break
    return algorithmic_bytes() * steps / el / 1e9, steps, el


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    warm = max(1, min(args.warmup, 2))
    time_oracle(0.0)  # builds + warms the oracle
    for _ in range(warm - 1):
        time_oracle(0.0)
    target = max(5.0, min(30.0, 0.05 * args.steps))
    gbs, steps, el = time_oracle(target)
    cores = oracle_threads()
    sample = (f"oracle matmul over the full {K}x{N} layer at M=1, {steps} steps in "
              f"{el:.1f} s (bounded sample of the benchmark's step count)")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": el / steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N,
                                        "bits": BITS, "group": GROUP, "symmetric": SYM},
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm

def run_wq(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    import synth
    import w4a16_decode_matmul_b200 as wq

    # one quantized layer, replicated into a pool larger than 4x L2
    W = synth.weight(N, K, seed=0).to(dev)
    base = wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM)
    del W
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    layer_bytes = base.nbytes
    pool_n = max(2, -(-4 * l2 // layer_bytes) + 1)
    pool = [wq.QuantizedWeight(base.codes.clone(), base.scales.clone(),
                               None if base.zeros is None else base.zeros.clone(),
                               N, K, BITS, GROUP, SYM) for _ in range(pool_n)]
    X = synth.activation(M, K, seed=1).to(dev)
    Y = torch.empty(M, N, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)

    def capture(count: int):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            wq.matmul(X, pool[0], out=Y, static_weights=True)  # warm the binding on this stream
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in range(count):
                    # the layer weights are static: each launch may start streaming
                    # them while the previous one finishes (programmatic dependent launch)
                    wq.matmul(X, pool[i % pool_n], out=Y, static_weights=True)
        return g

    steps = args.steps
    warm = max(args.warmup, 3)
    # The timed launches are replayed from CUDA graphs: one graph of exactly
    # `steps` launches when that is small, else a graph of one pool cycle
    # replayed `full` times plus one of the `rest`.  Every graph is replayed
    # before the timed region, so that no first-replay cost is timed.
    if steps <= GRAPH_MAX_LAUNCHES:
        graphs = [(capture(steps), 1)]
    else:
        full, rest = divmod(steps, pool_n)
        graphs = [(capture(pool_n), full)] + ([(capture(rest), 1)] if rest else [])
    g_cycle = capture(pool_n)            # for the per-replay distribution
    with torch.cuda.stream(stream):
        for g, _ in graphs:
            g.replay()
        for _ in range(max(1, -(-warm // pool_n))):
            g_cycle.replay()
    stream.synchronize()

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(f"GPU-{torch.cuda.get_device_properties(dev).uuid}") as clocks:
        with torch.cuda.stream(stream):
            # a short device-side wait ahead of the start event, so that the
            # host has queued every replay before the timed region begins
            torch.cuda._sleep(SLEEP_CYCLES)
            start.record(stream)
            for g, n in graphs:
                for _ in range(n):
                    g.replay()
            end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms_local = start.elapsed_time(end)
    ms = reduce_max(ms_local, dev)
    clk = clocks.summary()
    err = wq.get_device_error(dev)

    bytes_step = algorithmic_bytes()
    value = whole_job_gbs(bytes_step, steps, world, ms)
    per_launch_ms = ms_local / steps
    achieved = bytes_step / (per_launch_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peaks()
    traffic = None
    if os.path.exists(PROFILE_SUMMARY):
        prof = json.load(open(PROFILE_SUMMARY))
        if prof.get("kernel_source_hash") == kernel_source_hash():
            traffic = prof.get("dram_bytes_per_launch")

    # comparison points on the same GPU (not part of the timed region)
    extra = compare_points(wq, torch, dev, stream, pool, X, pool_n)
    extra["per_graph_distribution"] = graph_distribution(torch, dev, stream, g_cycle, pool_n)
    extra["warm_l2"] = warm_l2_point(wq, torch, dev, stream, pool[0], X)
    # the shipping launch mode (graph, static weights: each launch a
    # programmatic dependent of the previous one) against the dense graph
    extra["headline_vs_dense_speedup"] = round(
        extra["dense_bf16_gemv"]["us_per_layer"] / (per_launch_ms * 1e3), 3)
    extra["stream_read_ceiling"] = stream_ceiling(wq, torch, dev, stream, pool, pool_n)
    extra["stream_read_ceiling"]["fused_frac_of_ceiling"] = round(
        extra["stream_read_ceiling"]["us_per_layer"] / (per_launch_ms * 1e3), 4)

    # end to end through the public API: host X in, host Y out, every step
    e2e = measure_e2e(wq, torch, dev, pool, pool_n, args)

    # the prefill row (tensor cores), outside the timed region
    del pool, graphs, g_cycle
    prefill = prefill_points(wq, torch, dev)
    # the quantize rows: the benchmark layer, then every matrix of the model
    quant = quantize_points(wq, torch, dev, stream)
    model_quant = whole_model_quantize(wq, torch, dev, stream)
    q4k = q4k_point(wq, torch, dev, stream)
    w8 = w8_gemv_point(wq, torch, dev, stream)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world,
        "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": ms / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": M, "K": K, "N": N, "bits": BITS,
                   "group": GROUP, "symmetric": SYM, "parallelism": f"replicas{world}",
                   "l2": (f"rotating pool of {pool_n} weight copies "
                          f"({pool_n * layer_bytes / 1e6:.0f} MB, "
                          f"{pool_n * layer_bytes / l2:.1f}x the {l2 / 1e6:.0f} MB L2)"),
                   "timing": ("CUDA graphs (" + ("one graph of all steps" if steps <= GRAPH_MAX_LAUNCHES
                                                 else f"{pool_n}-launch cycles") +
                              ", each replayed once before timing), CUDA events on the launch "
                              "stream"),
                   "launch": "programmatic dependent launch (static weights)"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "peak_kind": f"{peak_kind} HBM copy"},
        "us_per_layer": round(per_launch_ms * 1e3, 3),
        "frac_of_nominal_8tbs": round(achieved / 8000.0, 4),
        "gpu_launches": steps,
        "clocks": clk,
        "e2e": e2e,
        "device_status": err,
        **extra,
        "prefill_tcgen05": prefill,
        "quantize_layer": quant,
        "quantize_whole_model": model_quant,
        "q4k_gemv": q4k,
        "w8a16_gemv": w8,
        "page2_h100_bandwidth_model": PAGE2_H100_CONTEXT,
    }
    if world == 1:
        cores = oracle_threads()
        gbs, st, el = time_oracle(8.0, threads=cores)
        gbs1, st1, el1 = time_oracle(6.0, threads=1)
        line["cpu_baseline"] = {
            "value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": (f"oracle matmul over the full {K}x{N} layer at M=1, {st} steps in "
                       f"{el:.1f} s on {cores} threads"),
            "single_thread": {"value": round(gbs1, 4), "unit": "GB/s", "cores": 1,
                              "sample": f"{st1} steps in {el1:.1f} s"}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def compare_points(wq, torch, dev, stream, pool, X, pool_n, reps: int = 50):
    """Dense bf16 GEMV (torch) and the unfused dequantize + GEMV on the same
    shape, with the same rotation over copies; microseconds per layer.  Each
    path is timed as one replay of a CUDA graph of `reps` calls (as the
    headline is), so that host launch costs do not enter; the fused path's
    eager time is reported beside it for information."""
    Wd = [torch.randn(N, K, device=dev, dtype=torch.bfloat16) for _ in range(
        max(2, -(-4 * torch.cuda.get_device_properties(dev).L2_cache_size // (N * K * 2)) + 1))]
    Wq_tmp = torch.empty(N, K, device=dev, dtype=torch.bfloat16)
    Y = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
    Yf = torch.empty(M, N, device=dev, dtype=torch.float32)

    def timed(fn, n):
        with torch.cuda.stream(stream):
            for i in range(3):
                fn(i)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            for i in range(n):
                fn(i)
            e.record(stream)
        torch.cuda.synchronize(dev)
        return s.elapsed_time(e) / n * 1e3

    def timed_graph(fn, n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for i in range(3):
                fn(i)
            stream.synchronize()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    fn(i)
            g.replay()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            g.replay()
            e.record(stream)
        torch.cuda.synchronize(dev)
        us = s.elapsed_time(e) / n * 1e3
        del g
        return us

    dense = lambda i: torch.matmul(X, Wd[i % len(Wd)].T, out=Y)
    unfused = lambda i: (wq.dequantize(pool[i % pool_n], out=Wq_tmp),
                         torch.matmul(X, Wq_tmp.T, out=Y))
    fused = lambda i: wq.matmul(X, pool[i % pool_n], out=Yf)
    dense_us = timed_graph(dense, reps)
    unfused_us = timed_graph(unfused, reps)
    fused_us = timed_graph(fused, reps)
    fused_eager_us = timed(fused, reps)
    dense_bytes = N * K * 2 + M * K * 2 + M * N * 2
    return {
        "dense_bf16_gemv": {"us_per_layer": round(dense_us, 3),
                            "gbs": round(dense_bytes / dense_us / 1e3, 1),
                            "how": f"torch.matmul bf16 [1,4096]x[4096,14336], CUDA graph of {reps} "
                                   f"calls over {len(Wd)} weight copies"},
        "unfused_dequant_then_gemv": {"us_per_layer": round(unfused_us, 3),
                                      "how": "wq_dequantize to bf16 then torch.matmul, same graph"},
        "fused_graph_us_per_layer": round(fused_us, 3),
        "fused_eager_us_per_layer": round(fused_eager_us, 3),
        "fused_vs_dense_speedup": round(dense_us / fused_us, 3),
        "speedup_how": ("dense ÷ fused, both as CUDA graphs of plain calls (no programmatic "
                        "dependent launch on either side)"),
    }


def graph_distribution(torch, dev, stream, graph, pool_n: int, reps: int = 60):
    """Microseconds per layer of single replays of the timed graph (pool_n
    launches each): p10 / median / p90 over `reps` replays."""
    times = []
    with torch.cuda.stream(stream):
        for _ in range(reps):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record(stream)
            graph.replay()
            e.record(stream)
            times.append((s, e))
    torch.cuda.synchronize(dev)
    us = sorted(s.elapsed_time(e) * 1e3 / pool_n for s, e in times)
    pick = lambda q: round(us[min(len(us) - 1, int(q * len(us)))], 3)
    return {"p10_us": pick(0.1), "median_us": pick(0.5), "p90_us": pick(0.9),
            "replays": reps, "launches_per_replay": pool_n}


def warm_l2_point(wq, torch, dev, stream, qw, X, count: int = 20, reps: int = 20):
    """The same graph-launched matmul on ONE weight copy (31 MB, resident in
    the L2 after the first launch): labelled warm-L2, not an HBM figure."""
    Y = torch.empty(M, N, dtype=torch.float32, device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        wq.matmul(X, qw, out=Y, static_weights=True)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(count):
                wq.matmul(X, qw, out=Y, static_weights=True)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    torch.cuda.synchronize(dev)
    us = s.elapsed_time(e) * 1e3 / (count * reps)
    return {"us_per_layer": round(us, 3), "gbs": round(algorithmic_bytes() / us / 1e3, 1),
            "how": "one weight copy, L2-resident: not an HBM number"}


def stream_ceiling(wq, torch, dev, stream, pool, pool_n, reps: int = 20):
    """The practical ceiling at this size: a read-only streaming kernel of
    the library over the same bytes (codes, scales, zeros of each pool copy),
    launched back to back from a CUDA graph with programmatic dependent
    launch, exactly like the timed matmul."""
    import ctypes
    lib = wq.lib
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.wq_internal_stream_read.argtypes = [vp, sz, vp, sz, vp, sz, vp, ctypes.c_int, vp]
    lib.wq_internal_stream_read.restype = ctypes.c_int
    lib.wq_internal_stream_read_out_bytes.argtypes = []
    lib.wq_internal_stream_read_out_bytes.restype = sz
    out = torch.empty(lib.wq_internal_stream_read_out_bytes() // 4, dtype=torch.int32, device=dev)

    def nbytes(t):
        return 0 if t is None else t.numel() * t.element_size()

    def launch(i):
        q = pool[i % pool_n]
        st = lib.wq_internal_stream_read(
            q.codes.data_ptr(), nbytes(q.codes), q.scales.data_ptr(), nbytes(q.scales),
            None if q.zeros is None else q.zeros.data_ptr(), nbytes(q.zeros),
            out.data_ptr(), 1, stream.cuda_stream)
        if st != 0:
            raise RuntimeError(f"wq_internal_stream_read: status {st}")

    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        launch(0)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for i in range(pool_n):
                launch(i)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    torch.cuda.synchronize(dev)
    us = s.elapsed_time(e) * 1e3 / (pool_n * reps)
    read = nbytes(pool[0].codes) + nbytes(pool[0].scales) + nbytes(pool[0].zeros)
    return {"us_per_layer": round(us, 3), "gbs": round(read / us / 1e3, 1),
            "bytes_per_layer": read,
            "how": "library read-only streaming kernel (16-byte loads, 4 CTAs x 512 threads "
                   "per SM) over each copy's codes+scales+zeros, CUDA graph of "
                   f"{pool_n} launches with programmatic dependent launch"}


def quantize_bytes(n: int, k: int, bits: int = BITS, group: int = GROUP, sym: bool = SYM) -> int:
    """Bytes the quantize pass must move: read W (binary16), write codes,
    scales and (asymmetric) zeros."""
    return 2 * n * k + n * k * bits // 8 + (n * k // group) * 2 * (1 if sym else 2)


def quantize_points(wq, torch, dev, stream, copies: int = 3, reps: int = 10):
    """wq_quantize on the benchmark layer (W [14336, 4096] binary16, 117 MB),
    rotating over `copies` different inputs so that the reads come from HBM."""
    import synth
    Ws = [synth.weight(N, K, seed=10 + i, device=dev) for i in range(copies)]
    outs = [wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM) for W in Ws]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        wq.quantize(Ws[0], bits=BITS, group=GROUP, symmetric=SYM, out=outs[0])
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for W, q in zip(Ws, outs):
                wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM, out=q)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    torch.cuda.synchronize(dev)
    us = s.elapsed_time(e) * 1e3 / (copies * reps)
    b = quantize_bytes(N, K)
    peak, kind = measured_peaks()
    return {"us": round(us, 2), "gbs": round(b / us / 1e3, 1), "bytes": b,
            "frac": round(b / us / 1e3 / peak, 4), "peak_kind": f"{kind} HBM copy",
            "how": f"CUDA graph over {copies} different W copies (117 MB each)"}


def whole_model_quantize(wq, torch, dev, stream, reps: int = 2):
    """Quantize every matrix of a Llama-8B-shaped model (32 layers x q, k, v,
    o, gate, up, down = 224 matrices, 6.98e9 binary16 weights, drawn on the
    GPU with seed 1000 * layer + projection): one CUDA graph of 224 quantize
    launches, timed as a whole.  The inputs (14 GB) are far larger than the
    L2."""
    import synth
    mats = synth.llama8b_matrices()
    Ws = [synth.weight(n, k, seed=seed, device=dev) for (_, _, _, n, k, seed) in mats]
    outs = [wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM) for W in Ws]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for W, q in zip(Ws, outs):
                wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM, out=q)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    torch.cuda.synchronize(dev)
    ms = s.elapsed_time(e) / reps
    b = sum(quantize_bytes(n, k) for (_, _, _, n, k, _) in mats)
    params = sum(n * k for (_, _, _, n, k, _) in mats)
    peak, kind = measured_peaks()
    del Ws, outs, g
    torch.cuda.empty_cache()
    return {"matrices": len(mats), "params": params, "ms": round(ms, 3),
            "gbs": round(b / ms / 1e6, 1), "bytes": b, "frac": round(b / ms / 1e6 / peak, 4),
            "peak_kind": f"{kind} HBM copy",
            "how": "CUDA graph of 224 wq_quantize launches, INT4 asymmetric group 128"}


def q4k_point(wq, torch, dev, stream, reps: int = 10):
    """The nested-superblock format (4.5 bits per weight) on the same layer:
    its quantize, and its fused M=1 matmul from a CUDA graph over a rotating
    pool of copies larger than 4x the L2 (plain launches)."""
    import synth
    W = synth.weight(N, K, seed=0).to(dev)
    base = wq.q4k_quantize(W)
    torch.cuda.synchronize(dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    nb = base.numel()
    pool_n = max(2, -(-4 * l2 // nb) + 1)
    pool = [base.clone() for _ in range(pool_n)]
    X = synth.activation(M, K, seed=1).to(dev)
    Y = torch.empty(M, N, dtype=torch.float32, device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        wq.q4k_matmul(X, pool[0], N, K, out=Y, static_weights=True)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for b in pool:
                wq.q4k_matmul(X, b, N, K, out=Y, static_weights=True)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    torch.cuda.synchronize(dev)
    us = s.elapsed_time(e) * 1e3 / (pool_n * reps)
    moved = nb + M * K * 2 + M * N * 4
    peak, kind = measured_peaks()
    return {"us_per_layer": round(us, 3), "gbs": round(moved / us / 1e3, 1),
            "bytes_per_layer": moved, "frac": round(moved / us / 1e3 / peak, 4),
            "peak_kind": f"{kind} HBM copy",
            "how": f"M=1, K={K}, N={N}, 144-byte superblocks (4.5 bits per weight), static "
                   f"weights (programmatic dependent launch), CUDA "
                   f"graph of {pool_n} launches over rotating copies"}


def w8_gemv_point(wq, torch, dev, stream, reps: int = 10):
    """The same layer with 8-bit codes (W8A16, asymmetric, group 128): the
    fused M=1 matmul from a CUDA graph over a rotating pool of copies larger
    than 4x the L2 (programmatic dependent launch); bytes moved and the
    fraction of the HBM copy peak."""
    import synth
    W = synth.weight(N, K, seed=0).to(dev)
    base = wq.quantize(W, bits=8, group=GROUP, symmetric=False)
    del W
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    pool_n = max(2, -(-4 * l2 // base.nbytes) + 1)
    pool = [wq.QuantizedWeight(base.codes.clone(), base.scales.clone(), base.zeros.clone(),
                               N, K, 8, GROUP, False) for _ in range(pool_n)]
    X = synth.activation(M, K, seed=1).to(dev)
    Y = torch.empty(M, N, dtype=torch.float32, device=dev)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        wq.matmul(X, pool[0], out=Y, static_weights=True)
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for q in pool:
                wq.matmul(X, q, out=Y, static_weights=True)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record(stream)
        for _ in range(reps):
            g.replay()
        e.record(stream)
    torch.cuda.synchronize(dev)
    us = s.elapsed_time(e) * 1e3 / (pool_n * reps)
    moved = algorithmic_bytes(bits=8)
    peak, kind = measured_peaks()
    return {"us_per_layer": round(us, 3), "gbs": round(moved / us / 1e3, 1),
            "bytes_per_layer": moved, "frac": round(moved / us / 1e3 / peak, 4),
            "peak_kind": f"{kind} HBM copy",
            "how": f"M=1, K={K}, N={N}, 8-bit asymmetric group 128, CUDA graph of {pool_n} "
                   "launches over rotating copies, programmatic dependent launch"}


def prefill_points(wq, torch, dev, reps: int = 8):
    """The prefill-shaped matmul (M in {512, 2048, 8192}, and the mid sizes 64
    and 256; K=4096, N=14336, INT4 asymmetric group 128) on the tensor cores
    next to a dense bf16 GEMM
    of the same shape (torch/cuBLAS); TFLOP/s = 2 M N K / time, and the
    fraction of the measured dense bf16 peak (burst)."""
    import synth
    qw = wq.quantize(synth.weight(N, K, seed=0).to(dev), bits=BITS, group=GROUP, symmetric=SYM)
    Wd = torch.randn(N, K, device=dev, dtype=torch.bfloat16)
    peak = measured_bf16_tflops()
    out = {}
    for m in (64, 256, 512, 2048, 8192):
        X = synth.activation(m, K, seed=3).to(dev)
        Y = torch.empty(m, N, device=dev, dtype=torch.float32)
        Yd = torch.empty(m, N, device=dev, dtype=torch.bfloat16)

        def timed(fn):
            for _ in range(2):
                fn()
            torch.cuda.synchronize(dev)
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            for _ in range(reps):
                fn()
            e.record()
            torch.cuda.synchronize(dev)
            return s.elapsed_time(e) / reps * 1e3

        us = timed(lambda: wq.matmul(X, qw, out=Y))
        dus = timed(lambda: torch.matmul(X, Wd.T, out=Yd))
        fl = 2.0 * m * N * K
        out[str(m)] = {"us": round(us, 1), "tflops": round(fl / us / 1e6, 1),
                       "frac_of_measured_bf16": round(fl / us / 1e6 / peak, 4),
                       "dense_bf16_us": round(dus, 1), "dense_bf16_tflops": round(fl / dus / 1e6, 1)}
        del X, Y, Yd
    return out


def measured_bf16_tflops():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"])
    return 1590.0


def _cudart():
    """ctypes handle on the CUDA runtime that torch loads (for plain
    cudaMemcpyAsync calls in the end-to-end loop), or None."""
    import ctypes
    import glob
    import nvidia
    for d in nvidia.__path__:
        for path in sorted(glob.glob(os.path.join(d, "cuda_runtime", "lib", "libcudart.so*"))):
            try:
                rt = ctypes.CDLL(path)
            except OSError:
                continue
            rt.cudaMemcpyAsync.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                           ctypes.c_int, ctypes.c_void_p]
            rt.cudaMemcpyAsync.restype = ctypes.c_int
            rt.cudaStreamSynchronize.argtypes = [ctypes.c_void_p]
            rt.cudaStreamSynchronize.restype = ctypes.c_int
            rt.cudaEventCreateWithFlags.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_uint]
            rt.cudaEventCreateWithFlags.restype = ctypes.c_int
            rt.cudaEventRecord.argtypes = [ctypes.c_void_p, ctypes.c_void_p]
            rt.cudaEventRecord.restype = ctypes.c_int
            rt.cudaEventSynchronize.argtypes = [ctypes.c_void_p]
            rt.cudaEventSynchronize.restype = ctypes.c_int
            rt.cudaEventDestroy.argtypes = [ctypes.c_void_p]
            rt.cudaEventDestroy.restype = ctypes.c_int
            return rt
    return None


def measure_e2e(wq, torch, dev, pool, pool_n, args):
    """End to end through the C ABI with host buffers, pipelined as a
    serving loop would run it: every step copies its X from pinned host
    memory to the device (cudaMemcpyAsync), calls wq_matmul and copies its
    Y back to pinned host memory; steps alternate between two streams with
    four buffer slots, and before a slot is reused the host waits for that
    step's Y and reads it.  Everything is inside the timed region (wall
    clock, max with the device events); at the end every slot's Y is
    checked against a device result of the same product."""
    import ctypes
    import synth
    lib = wq.lib
    rt = _cudart()
    depth, nstreams = 4, 2
    x_host = synth.activation(M, K, seed=1)
    Xh = [x_host.clone().pin_memory() for _ in range(depth)]
    Yh = [torch.empty(M, N, dtype=torch.float32).pin_memory() for _ in range(depth)]
    Xd = [torch.empty(M, K, dtype=torch.bfloat16, device=dev) for _ in range(depth)]
    Yd = [torch.empty(M, N, dtype=torch.float32, device=dev) for _ in range(depth)]
    streams = [torch.cuda.Stream(dev) for _ in range(nstreams)]
    handles = [ctypes.c_void_p(st.cuda_stream) for st in streams]
    wss = [wq.workspace(dev, st.cuda_stream) for st in streams]
    vp = ctypes.c_void_p
    # per-slot completion events (raw runtime events when the runtime is at
    # hand: cheaper per step than torch's) and numpy views of the host Y
    if rt is not None:
        events = []
        for _ in range(depth):
            ev = vp()
            if rt.cudaEventCreateWithFlags(ctypes.byref(ev), 2) != 0:  # cudaEventDisableTiming
                raise RuntimeError("cudaEventCreateWithFlags failed")
            events.append(ev)
        record = lambda slot, si: rt.cudaEventRecord(events[slot], handles[si])
        wait_slot = lambda slot: rt.cudaEventSynchronize(events[slot])
    else:
        events = [torch.cuda.Event() for _ in range(depth)]
        record = lambda slot, si: events[slot].record(streams[si])
        wait_slot = lambda slot: events[slot].synchronize()
    y_views = [y.numpy() for y in Yh]
    x_bytes, y_bytes = M * K * 2, M * N * 4

    def call(i, slot, si):
        q = pool[i % pool_n]
        return (vp(Xd[slot].data_ptr()), M, vp(q.codes.data_ptr()), vp(q.scales.data_ptr()),
                None if q.zeros is None else vp(q.zeros.data_ptr()), N, K, BITS, GROUP, int(SYM),
                vp(Yd[slot].data_ptr()), wq.WQ_OUT_F32, vp(wss[si].data_ptr()), wss[si].numel(),
                0, handles[si])

    calls = [[call(i, i % depth, (i % depth) % nstreams) for i in range(pool_n * depth)]]
    reads = [0.0]

    def step(i):
        slot = i % depth
        si = slot % nstreams          # a slot always uses the same stream
        h, st = handles[si], streams[si]
        if i >= depth:
            wait_slot(slot)           # step i - depth's Y is on the host: read it
            reads[0] += float(y_views[slot][0, 0])
        if rt is not None:
            rt.cudaMemcpyAsync(vp(Xd[slot].data_ptr()), vp(Xh[slot].data_ptr()), x_bytes, 1, h)
        else:
            with torch.cuda.stream(st):
                Xd[slot].copy_(Xh[slot], non_blocking=True)
        c = calls[0][i % len(calls[0])]
        status = lib.wq_matmul(*c)
        if status != 0:
            raise wq.WQError(status, "wq_matmul")
        if rt is not None:
            rt.cudaMemcpyAsync(vp(Yh[slot].data_ptr()), vp(Yd[slot].data_ptr()), y_bytes, 2, h)
        else:
            with torch.cuda.stream(st):
                Yh[slot].copy_(Yd[slot], non_blocking=True)
        record(slot, si)

    def drain(last):
        for i in range(max(0, last - depth), last):
            wait_slot(i % depth)
            reads[0] += float(y_views[i % depth][0, 0])

    steps = max(200, min(5000, args.steps))
    steps -= steps % (pool_n * depth)  # whole cycles: every weight copy and slot alike
    steps = max(steps, pool_n * depth)
    with torch.cuda.device(dev):
        for i in range(2 * depth):
            step(i)
        drain(2 * depth)
        torch.cuda.synchronize(dev)
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        s.record(streams[0])
        for i in range(steps):
            step(i)
        drain(steps)
        for st in streams[1:]:
            streams[0].wait_stream(st)
        e.record(streams[0])
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - t0
    ref = wq.matmul(x_host.to(dev), pool[0])
    torch.cuda.synchronize(dev)
    checked = all(torch.equal(Yh[j], ref.cpu()) for j in range(depth))
    if rt is not None:
        for ev in events:
            rt.cudaEventDestroy(ev)
    ms = reduce_max(max(s.elapsed_time(e), wall * 1e3), dev)
    _, world, _ = dist_env()
    return {"value": round(whole_job_gbs(algorithmic_bytes(), steps, world, ms), 3),
            "unit": "GB/s", "h2d_bytes_per_step": x_bytes, "d2h_bytes_per_step": y_bytes,
            "steps": steps, "us_per_step": round(ms / steps * 1e3, 3), "results_checked": checked,
            "how": ("C ABI wq_matmul per step between cudaMemcpyAsync of X (pinned host -> "
                    "device) and of Y (device -> pinned host); 4 buffer slots over 2 streams, "
                    "the host waits for and reads each step's Y before reusing its slot")}


def ncu_case(which: str = "decode"):
    """Small, self-contained launch sequences for ncu captures (no timing):

    decode   -- quantize the benchmark layer, 8 fused decode matmuls (M=1),
                then 2 prefill matmuls (M=2048) on it;
    traffic  -- the same layer through the three paths page 2 "实现" compares,
                3 launches each: the fused matmul; the unfused path
                (dequantize to bf16, then a cuBLAS bf16 GEMV); the dense bf16
                GEMV on a bf16 weight of the same shape;
    prefill  -- 2 prefill matmuls at M=2048;
    quantize -- 3 quantize launches over 3 different 117 MB layers;
    q4k      -- superblock quantize, then 4 superblock decode matmuls."""
    import torch
    import synth
    import w4a16_decode_matmul_b200 as wq
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    W = synth.weight(N, K, seed=0).to(dev)
    X = synth.activation(M, K, seed=1).to(dev)
    Y = torch.empty(M, N, dtype=torch.float32, device=dev)
    if which in ("decode", "traffic", "prefill"):
        qw = wq.quantize(W, bits=BITS, group=GROUP, symmetric=SYM)
    if which == "decode":
        for _ in range(8):
            wq.matmul(X, qw, out=Y)
    if which in ("decode", "prefill"):
        Xp = synth.activation(2048, K, seed=2).to(dev)
        Yp = torch.empty(2048, N, dtype=torch.float32, device=dev)
        for _ in range(2):
            wq.matmul(Xp, qw, out=Yp)
    if which == "traffic":
        Wt = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
        Wd = W.to(torch.bfloat16)
        Yb = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            wq.matmul(X, qw, out=Y)
        for _ in range(3):
            wq.dequantize(qw, out=Wt)
            torch.matmul(X, Wt.T, out=Yb)
        for _ in range(3):
            torch.matmul(X, Wd.T, out=Yb)
    if which == "quantize":
        Ws = [synth.weight(N, K, seed=10 + i, device=dev) for i in range(3)]
        for Wi in Ws:
            wq.quantize(Wi, bits=BITS, group=GROUP, symmetric=SYM)
    if which == "q4k":
        blocks = wq.q4k_quantize(W)
        for _ in range(4):
            wq.q4k_matmul(X, blocks, N, K, out=Y)
    torch.cuda.synchronize(dev)
    assert wq.get_device_error(dev) == 0
    print(f"ncu case {which} ok")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200000)
    ap.add_argument("--warmup", type=int, default=2000)
    ap.add_argument("--impl", choices=["wq", "reference"], default="wq")
    ap.add_argument("--ncu-case", nargs="?", const="decode", default=None,
                    choices=["decode", "traffic", "prefill", "quantize", "q4k"],
                    help="no timing: a short launch sequence for ncu captures (see ncu_case)")
    args = ap.parse_args(argv)
    if args.ncu_case:
        return ncu_case(args.ncu_case)
    if args.impl == "reference":
        return run_reference(args)
    return run_wq(args)


if __name__ == "__main__":
    sys.exit(main())
