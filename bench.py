#!/usr/bin/env python
"""Benchmark of the W4A16 hot path on B200.

Headline (``value``): decode GEMM HBM throughput at Llama-3-8B linear-layer
shapes, M = 1 -- one step = the four fused dequantize-matmul calls
(qkv 4096->6144, o_proj 4096->4096, gate_up 4096->28672, down 14336->4096) on
bf16 activations with packed uint4 weights resident in HBM.  Throughput is
algorithmic bytes (packed codes + fp16 scale/zero + X + fp32 Y) per second.

Also reported on the same JSON line:
  * roofline of the dominant kernel (gate_up): its average launch duration,
    from CUDA events around a CUDA graph of back-to-back gate_up launches over
    the same rotating weight copies;
  * e2e: the same metric through the C ABI's host-buffer entry point
    (pinned X in, fp32 Y out, copies inside the timed region);
  * e2e_batched: the same through the batched host-buffer entry point (the
    step's four independent matmuls in one call: one copy in, one copy out);
  * quantize: the quantize+pack kernel on the same four layers (fp32 W in);
  * prefill: TFLOP/s of the tensor-core path at Llama-3-70B shapes, M = 8192;
  * cpu_baseline: the oracle (plain C, one core) on a bounded sample.

Multi-GPU: each rank runs its own copy of the step (independent problems, no
collective on the data path): weak scaling, value = all ranks' bytes / max time.

``--impl reference`` times the oracle alone on the host (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from weight_only_int4_w4_b200 import synthetic  # noqa: E402

METRIC = "W4A16 GEMM: decode HBM GB/s and prefill TFLOP/s vs B200 roofline, 1 GPU"
G = 128
LAYERS = list(synthetic.SHAPES_8B)  # qkv, o_proj, gate_up, down
DOMINANT = "gate_up"
N_COPIES = 5  # weight copies rotated across steps: 5 x 116 MB > 4 x L2 (126 MB)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# Nominal B200 figures, reported beside the measured ones: ~8 TB/s HBM3e and
# 2.25 PFLOP/s dense bf16 (NVIDIA's per-GPU dense figure).
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


def gemm_bytes(M, N, K):
    """Algorithmic bytes of one fused call: packed codes + fp16 scale & zero + X (bf16) + Y (fp32)."""
    return N * K // 2 + 4 * N * (K // G) + 2 * M * K + 4 * M * N


def quant_bytes(N, K):
    """fp32 W in, packed codes + fp16 scale & zero out."""
    return 4 * N * K + N * K // 2 + 4 * N * (K // G)


KERNEL_SOURCES = {"gemv_mma_gate_up_m1": ("common.cuh", "gemv_mma.cu")}  # files that define the kernel


def kernel_source_hash(kernel_key="gemv_mma_gate_up_m1"):
    h = hashlib.sha256()
    d = os.path.join(ROOT, "weight_only_int4_w4_b200", "csrc")
    for f in KERNEL_SOURCES[kernel_key]:
        h.update(open(os.path.join(d, f), "rb").read())
    return h.hexdigest()[:16]


def committed_traffic(kernel_key):
    """DRAM bytes per launch from the committed ncu summary, if it matches today's kernels."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        e = t.get(kernel_key)
        if e and e.get("source_hash") == kernel_source_hash(kernel_key):
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.dev = device_index

    def __enter__(self):
        try:
            uuid = None
            try:
                uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
                if not uuid.startswith("GPU-"):
                    uuid = "GPU-" + uuid
            except Exception:
                pass
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
            if uuid:
                cmd += ["-i", uuid]
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not getattr(self, "out", ""):
            return None
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[0]))
                mx = float(f[1])
            except ValueError:
                continue
            for name, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def _all_reduce(v, op):
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(v, world):
    """Slowest rank's time: the job is done when every rank is done."""
    return v if world == 1 else _all_reduce(v, torch.distributed.ReduceOp.MAX)


def sum_over_ranks(v, world):
    """Total work of all ranks (weak scaling: each rank runs its own copy of the step)."""
    return v if world == 1 else _all_reduce(v, torch.distributed.ReduceOp.SUM)


def job_throughput(bytes_per_rank, ms_per_rank, world):
    """Whole-job GB/s: all ranks' bytes over the slowest rank's device time."""
    ms = max_over_ranks(ms_per_rank, world)
    return sum_over_ranks(bytes_per_rank, world) / (ms * 1e-3) / 1e9, ms


def decode_config(world):
    return {"workload": "decode_8b: Llama-3-8B qkv/o_proj/gate_up/down, M=1, bf16 X ~N(0,1), "
                        "W ~N(0,0.02) with 0.1% N(0,0.4) outliers, uint4 G=128",
            "global_batch": world, "seq_len": 1, "parallelism": f"replicas{world}"}


# ----------------------------------------------------------------------------- CPU oracle
def cpu_oracle_step(rows_per_layer):
    """One oracle decode step on a sample: for each 8B layer, dequantize `rows_per_layer`
    rows of pre-quantized weights and do the fp64 matmul with X (M=1).  Returns bytes."""
    import oracle  # test/bench-only: the CPU baseline leg
    total = 0
    for name in LAYERS:
        K, N = synthetic.SHAPES_8B[name]
        key = (name, rows_per_layer)
        if key not in _ORACLE_CACHE:
            rows = list(range(min(rows_per_layer, N)))
            W = synthetic.weight_rows(K, N, 0.02, 0.001, ("decode_8b", name), rows=rows).numpy()
            X = synthetic.activations(1, K, "bf16", ("decode_8b", name)).float().numpy()
            _ORACLE_CACHE[key] = (oracle.quantize(W), X)
        (codes, sc, zp), X = _ORACLE_CACHE[key]
        What = oracle.dequant(codes, sc, zp)
        oracle.gemm(X, What)
        total += gemm_bytes(1, codes.shape[0], K)
    return total


_ORACLE_CACHE = {}


def time_cpu_oracle(budget_s=12.0, rows_per_layer=512):
    cpu_oracle_step(rows_per_layer)  # build caches
    t0 = time.perf_counter()
    nbytes, reps = 0, 0
    while time.perf_counter() - t0 < budget_s:
        nbytes += cpu_oracle_step(rows_per_layer)
        reps += 1
    dt = time.perf_counter() - t0
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{rows_per_layer} output rows of each of the 4 Llama-3-8B layers (dequant + fp64 matmul, M=1), "
                      f"{reps} repetitions in {dt:.1f} s on one host core"}


def _oracle_worker(rows, budget_s):
    """One process of the all-cores oracle timing: its own row slice of every layer, looped
    for budget_s seconds after a warm-up; returns the algorithmic bytes it covered and its time."""
    torch.set_num_threads(1)  # one core per process
    cpu_oracle_step(rows)
    t0 = time.perf_counter()
    nbytes = 0
    while time.perf_counter() - t0 < budget_s:
        nbytes += cpu_oracle_step(rows)
    return nbytes, time.perf_counter() - t0


def _oracle_70b_worker(part, parts):
    """One process of the whole-stack oracle estimate: rows [part/parts] of each Llama-3-70B
    layer shape and of lm_head, dequant + fp64 matmul at M=1.  The codes, scales and zeros
    are drawn uniformly (the oracle's time does not depend on their values).  Returns the
    algorithmic bytes and seconds of its slice of one layer set, and of lm_head."""
    import numpy as np
    import oracle  # test/bench-only: the CPU baseline leg
    torch.set_num_threads(1)
    rng = np.random.default_rng(synthetic.seed_of("oracle70b", part, parts) % (2 ** 62))

    def one(K, N):
        n = N * (part + 1) // parts - N * part // parts
        if n == 0:
            return 0, 0.0
        codes = rng.integers(0, 16, size=(n, K), dtype=np.uint8)
        sc = (0.001 + 0.003 * rng.random((n, K // G), dtype=np.float32)).astype(np.float16)
        zp = rng.integers(0, 16, size=(n, K // G)).astype(np.float16)
        X = rng.standard_normal((1, K), dtype=np.float32)
        t0 = time.perf_counter()
        oracle.gemm(X, oracle.dequant(codes, sc, zp))
        return gemm_bytes(1, n, K), time.perf_counter() - t0

    layer = [one(K, N) for K, N in synthetic.SHAPES_70B.values()]
    head = one(*synthetic.LM_HEAD_70B)
    return sum(b for b, _ in layer), sum(t for _, t in layer), head[0], head[1]


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def time_cpu_oracle_all_cores(budget_s=10.0, rows_per_layer=512):
    """The oracle on the host cores (up to 32): one spawned process per core, each on its own
    512-row sample of each layer (independent rows, as the oracle computes them one by one)."""
    import multiprocessing as mp
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    cores = min(cores, 32)  # bounds the start-up cost (each process imports torch)
    ctx = mp.get_context("spawn")
    with ctx.Pool(cores) as pool:
        res = pool.starmap(_oracle_worker, [(rows_per_layer, budget_s)] * cores)
        res70 = pool.starmap(_oracle_70b_worker, [(i, cores) for i in range(cores)])
    nbytes = sum(r[0] for r in res)
    dt = max(r[1] for r in res)
    eight_b = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{cores} processes, each {rows_per_layer} output rows of each of the 4 Llama-3-8B layers "
                         f"(dequant + fp64 matmul, M=1) for {budget_s:.0f} s; CPU: {cpu_model()}"}
    # Whole 70B stack at M=1: one full layer set and lm_head measured, the layers extrapolated x80.
    n_layers = synthetic.N_LAYERS_70B
    step_bytes = n_layers * sum(r[0] for r in res70) + sum(r[2] for r in res70)
    step_s = max(n_layers * r[1] + r[3] for r in res70)
    stack = {"value": step_bytes / step_s / 1e9, "unit": "GB/s", "ms_per_step": step_s * 1e3, "cores": cores,
             "kind": "oracle",
             "sample": f"one full Llama-3-70B layer set (qkv, o_proj, gate_up, down) and lm_head at M=1, rows split "
                       f"over {cores} processes, dequant + fp64 matmul; the step time extrapolates the layer set "
                       f"x{n_layers} plus lm_head"}
    return eight_b, stack


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    rows = 256
    for _ in range(args.warmup):
        cpu_oracle_step(rows)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += cpu_oracle_step(rows)
    dt = time.perf_counter() - t0
    v = nbytes / dt / 1e9
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32xu4->f64", "data": "synthetic",
        "config": decode_config(world),
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"{rows} output rows of each of the 4 Llama-3-8B layers per step (dequant + fp64 matmul, M=1)"},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ----------------------------------------------------------------------------- GPU legs
def build_decode_state(w4, dev):
    gen = torch.Generator(device=dev)
    layers = {}
    for name in LAYERS:
        K, N = synthetic.SHAPES_8B[name]
        gen.manual_seed(synthetic.seed_of("bench", "decode_8b", name) % (2 ** 62))
        W = torch.randn((N, K), generator=gen, device=dev, dtype=torch.float32) * 0.02
        mask = torch.rand((N, K), generator=gen, device=dev) < 0.001
        W = torch.where(mask, torch.randn((N, K), generator=gen, device=dev) * synthetic.OUTLIER_STD, W)
        packed, scales, zeros = w4.w4_quantize(W)
        del W, mask
        X = (torch.randn((1, K), generator=gen, device=dev)).to(torch.bfloat16)
        copies = [(packed, scales, zeros)] + [(packed.clone(), scales.clone(), zeros.clone()) for _ in range(N_COPIES - 1)]
        Y = torch.empty((1, N), dtype=torch.float32, device=dev)
        ws_bytes = w4.w4a16_gemm_workspace_size(1, N, K)
        ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        layers[name] = dict(K=K, N=N, X=X, copies=copies, Y=Y, ws=ws)
    torch.cuda.synchronize()
    return layers


def _graph_of(fn, steps, warmup, stream):
    with torch.cuda.stream(stream):
        for i in range(warmup):
            fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            fn(i)
    with torch.cuda.stream(stream):  # warm replay of the graph itself
        g.replay()
    torch.cuda.synchronize()
    return g


def _replay_timed(g, stream):
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def decode_leg(w4, layers, steps, warmup, world):
    """The timed steps: `steps` decode steps (4 fused calls each) in one CUDA graph."""
    stream = torch.cuda.Stream()

    def step(i):
        for name in LAYERS:
            L = layers[name]
            packed, scales, zeros = L["copies"][i % N_COPIES]
            w4.w4a16_gemm(L["X"], packed, scales, zeros, out=L["Y"], ws=L["ws"])

    g = _graph_of(step, steps, warmup, stream)
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        ms = _replay_timed(g, stream)
    barrier(world)
    # 20 more replays of the same graph, each timed alone, for the spread of the
    # step time (the value is the single timed region of exactly `steps` steps).
    reps = sorted(_replay_timed(g, stream) / steps for _ in range(20))
    del g
    repeats = {"n": 20, "steps_each": steps,
               "median_ms_per_step": round(max_over_ranks(statistics.median(reps), world), 5),
               "min_ms_per_step": round(reps[0], 5), "max_ms_per_step": round(reps[-1], 5)}
    return ms, clk.summary(), repeats


def dominant_leg(w4, layers, launches, warmup):
    """Average launch duration of the dominant kernel (gate_up, M=1): `launches`
    launches over the rotating weight copies in one CUDA graph, timed with events
    on the stream they run on."""
    stream = torch.cuda.Stream()
    L = layers[DOMINANT]

    def one(i):
        packed, scales, zeros = L["copies"][i % N_COPIES]
        w4.w4a16_gemm(L["X"], packed, scales, zeros, out=L["Y"], ws=L["ws"])

    g = _graph_of(one, launches, warmup, stream)
    ms = _replay_timed(g, stream)
    del g
    return ms / launches


def e2e_leg(w4, layers, steps, warmup, world):
    """Same step through the C ABI's host-buffer entry point: pinned X in, Y out, per
    layer, enqueued without a wait (w4a16_gemm_host_async); the host waits for the
    stream once per step, after the last layer's output copy."""
    host = {}
    for name in LAYERS:
        L = layers[name]
        host[name] = (L["X"].cpu().pin_memory(), torch.empty((1, L["N"]), dtype=torch.float32).pin_memory())
    stream = torch.cuda.Stream()

    def step(i):
        for name in LAYERS:
            L = layers[name]
            packed, scales, zeros = L["copies"][i % N_COPIES]
            Xh, Yh = host[name]
            w4.w4a16_gemm_host(Xh, L["X"], packed, scales, zeros, Yh, L["Y"], ws=L["ws"], stream=stream, wait=False)
        stream.synchronize()  # the step's outputs are in host memory

    for i in range(warmup):
        step(i)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    h2d = sum(2 * layers[n]["K"] for n in LAYERS)
    d2h = sum(4 * layers[n]["N"] for n in LAYERS)
    return a.elapsed_time(b), h2d, d2h


def e2e_batch_leg(w4, layers, steps, warmup, world):
    """The step's four independent matmuls in one call of the batched host-buffer entry
    (w4a16_gemm_host_batch_async): the four pinned X in one copy, the four matmuls, the
    four fp32 Y back in one copy; the host waits for the stream once per step."""
    xo, yo, offs = 0, 0, {}
    for name in LAYERS:
        L = layers[name]
        offs[name] = (xo, yo)
        xo += -(-2 * L["K"] // 16) * 16
        yo += -(-4 * L["N"] // 16) * 16
    Xh = torch.zeros(xo, dtype=torch.uint8).pin_memory()
    for name in LAYERS:
        x = layers[name]["X"].cpu().contiguous().view(torch.uint8).reshape(-1)
        Xh[offs[name][0]:offs[name][0] + x.numel()] = x
    Yh = torch.empty(yo, dtype=torch.uint8).pin_memory()
    dev = layers[LAYERS[0]]["X"].device
    Xd = torch.empty(xo, dtype=torch.uint8, device=dev)
    Yd = torch.empty(yo, dtype=torch.uint8, device=dev)
    ws = max((layers[n]["ws"] for n in LAYERS), key=lambda t: t.numel())
    batches = []
    for c in range(N_COPIES):
        items = []
        for name in LAYERS:
            L = layers[name]
            packed, scales, zeros = L["copies"][c]
            items.append(dict(M=1, N=L["N"], K=L["K"], packed=packed, scales=scales, zeros=zeros,
                              x_offset=offs[name][0], y_offset=offs[name][1]))
        batches.append(w4.gemm_batch(items))
    stream = torch.cuda.Stream()

    def step(i):
        w4.w4a16_gemm_host_batch(batches[i % N_COPIES], Xh, Xd, Yh, Yd, ws=ws, stream=stream, wait=False)
        stream.synchronize()  # the step's outputs are in host memory

    for i in range(warmup):
        step(i)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(steps):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    return a.elapsed_time(b), xo, yo


def quantize_leg(w4, steps=5):
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    Ws = []
    for name in LAYERS:
        K, N = synthetic.SHAPES_8B[name]
        gen.manual_seed(synthetic.seed_of("bench", "quant", name) % (2 ** 62))
        Ws.append(torch.randn((N, K), generator=gen, device=dev) * 0.02)
    outs = [(torch.empty((W.shape[0], W.shape[1] // 2), dtype=torch.uint8, device=dev),
             torch.empty((W.shape[0], W.shape[1] // G), dtype=torch.float16, device=dev),
             torch.empty((W.shape[0], W.shape[1] // G), dtype=torch.float16, device=dev)) for W in Ws]
    import ctypes
    lib = w4.lib

    def run():
        s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for W, (p, sc, z) in zip(Ws, outs):
            st = lib.w4_quantize(ctypes.c_void_p(W.data_ptr()), 0, None, W.shape[0], W.shape[1], G,
                                 ctypes.c_void_p(p.data_ptr()), ctypes.c_void_p(sc.data_ptr()),
                                 ctypes.c_void_p(z.data_ptr()), None, s)
            assert st == 0
    run()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        run()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / steps
    nbytes = sum(quant_bytes(W.shape[0], W.shape[1]) for W in Ws)
    del Ws, outs
    torch.cuda.empty_cache()
    return ms, nbytes


PREFILL_MS = (512, 2048, 8192)


def prefill_leg(w4, bf16_peak, Ms=PREFILL_MS):
    """Tensor-core GEMM at the Llama-3-70B shapes for every prefill M: per layer TFLOP/s and
    the fraction of the measured (burst) and nominal dense bf16 peaks; each layer's weights
    are quantized once and reused for all M.  Launches are timed back to back with events
    on the launching stream, after one warm-up launch."""
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    steps_for = {512: 20, 2048: 8, 8192: 3}
    per = {M: {} for M in Ms}
    tot = {M: [0.0, 0.0] for M in Ms}
    Xall = None
    for name, (K, N) in synthetic.SHAPES_70B.items():
        gen.manual_seed(synthetic.seed_of("bench", "prefill", name) % (2 ** 62))
        W = torch.randn((N, K), generator=gen, device=dev) * 0.015
        packed, scales, zeros = w4.w4_quantize(W)
        del W
        Xall = torch.randn((max(Ms), K), generator=gen, device=dev).to(torch.bfloat16)
        for M in Ms:
            X = Xall[:M]
            Y = torch.empty((M, N), dtype=torch.float32, device=dev)
            ws = w4.workspace(M, N, K, dev)
            w4.w4a16_gemm(X, packed, scales, zeros, out=Y, ws=ws)
            torch.cuda.synchronize()
            steps = steps_for.get(M, 3)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(steps):
                w4.w4a16_gemm(X, packed, scales, zeros, out=Y, ws=ws)
            b.record()
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / steps
            flop = 2.0 * M * N * K
            tf = flop / (ms * 1e-3) / 1e12
            per[M][name] = {"tflops": round(tf, 1), "us_per_call": round(ms * 1e3, 2),
                            "frac": round(tf / bf16_peak, 4), "frac_nominal": round(tf / NOMINAL_BF16_TFLOPS, 4)}
            tot[M][0] += flop
            tot[M][1] += ms
            del Y
        del packed, scales, zeros, Xall
        torch.cuda.empty_cache()
    out = {}
    for M in Ms:
        tf = tot[M][0] / (tot[M][1] * 1e-3) / 1e12
        out[f"M{M}"] = {"tflops": round(tf, 1), "ms_per_step": round(tot[M][1], 3), "frac": round(tf / bf16_peak, 4),
                        "frac_nominal": round(tf / NOMINAL_BF16_TFLOPS, 4), "per_layer": per[M]}
    return out


def stack70b_leg(w4, replays=3):
    """Whole-model 70B decode step: quantize the 80-layer stack + lm_head on the device, then
    one step through all 321 linear layers at M=1 and at M=16, each captured in a CUDA graph."""
    from weight_only_int4_w4_b200 import stack70b
    layers, q_ms, q_bytes = stack70b.build(w4)
    out = {"workload": "Llama-3-70B stack: 80 x (qkv, o_proj, gate_up, down) + lm_head, "
                       "69.50 G params, 36.92 GB packed, W ~N(0,0.015), bf16 X ~N(0,1)",
           "quantize": {"value": round(q_bytes / (q_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                        "ms_total": round(q_ms, 2), "bytes": q_bytes,
                        "frac": round(q_bytes / (q_ms * 1e-3) / 1e9 / peaks()[0], 4),
                        "timing": "summed device time of the 321 quantize launches; outputs allocated "
                                  "before each launch's events"}}
    hbm_peak = peaks()[0]
    for M in (1, 16):
        X, Y, ws = stack70b.step_buffers(w4, layers, M)
        stream = torch.cuda.Stream()
        g = _graph_of(lambda i: stack70b.run_step(w4, layers, X, Y, ws), 1, 1, stream)
        ms = min(_replay_timed(g, stream) for _ in range(replays))
        del g
        nbytes = stack70b.step_bytes(layers, M)
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[f"decode_m{M}"] = {"us_per_step": round(ms * 1e3, 1), "GB/s": round(gbs, 1),
                                "bytes_per_step": nbytes, "roofline_frac": round(gbs / hbm_peak, 4),
                                "roofline_frac_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                                "launches": len(layers)}
        del X, Y, ws
    del layers
    torch.cuda.empty_cache()
    return out


def verify_leg(w4, Ms=(4, 8, 16, 32, 48, 64), steps=20):
    """Speculative-verification / small-batch decode: the four Llama-3-8B layers with the AWQ
    scale folded in, at each M; two weight copies per layer rotate (232 MB > L2); each M's
    steps are captured in one CUDA graph."""
    dev = torch.device("cuda")
    gen = torch.Generator(device=dev)
    layers = []
    for name in LAYERS:
        K, N = synthetic.SHAPES_8B[name]
        s = synthetic.awq_scale(K, ("bench", "verify", name)).to(dev)
        copies = []
        for c in range(2):
            gen.manual_seed(synthetic.seed_of("bench", "verify", name, c) % (2 ** 62))
            W = torch.randn((N, K), generator=gen, device=dev) * 0.02
            copies.append(w4.w4_quantize(W, s))
            del W
        layers.append((K, N, s, copies))
    stream = torch.cuda.Stream()
    out = {}
    for M in Ms:
        bufs = []
        for K, N, s, copies in layers:
            X = torch.randn((M, K), generator=gen, device=dev).to(torch.bfloat16)
            bufs.append((X, torch.empty((M, N), dtype=torch.float32, device=dev), w4.workspace(M, N, K, dev)))

        def step(i):
            for (K, N, s, copies), (X, Y, ws) in zip(layers, bufs):
                packed, scales, zeros = copies[i % 2]
                w4.w4a16_gemm(X, packed, scales, zeros, s, out=Y, ws=ws)

        g = _graph_of(step, steps, 3, stream)
        ms = _replay_timed(g, stream) / steps
        del g
        nbytes = sum(gemm_bytes(M, N, K) + 4 * K for K, N, _, _ in layers)
        flop = sum(2.0 * M * N * K for K, N, _, _ in layers)
        hbm_peak, bf16_peak = peaks()[0], peaks()[1]
        t_roof_us = max(nbytes / (hbm_peak * 1e9), flop / (bf16_peak * 1e12)) * 1e6
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[f"M{M}"] = {"us_per_step": round(ms * 1e3, 2), "GB/s": round(gbs, 1),
                        "roofline": {"bound": "hbm", "frac": round(gbs / hbm_peak, 4),
                                     "frac_nominal": round(gbs / NOMINAL_HBM_GBS, 4),
                                     "roofline_us": round(t_roof_us, 2),
                                     "frac_of_roofline_time": round(t_roof_us / (ms * 1e3), 4)}}
    out["workload"] = ("verify_8b: qkv/o_proj/gate_up/down with AWQ s, bf16 X, M = batch x (draft 5 + 1); "
                       "M <= 8 on the decode kernel, above on the tensor-core kernel")
    del layers
    torch.cuda.empty_cache()
    return out


def outlier_leg(w4, launches=60):
    """Decode GEMM with the dense + sparse outlier split (0.1% of the weights in fp16 CSR) on the
    Llama-3-8B gate_up shape at M=1, three weight copies rotated (188 MB > L2), in one CUDA graph."""
    dev = torch.device("cuda")
    K, N = synthetic.SHAPES_8B["gate_up"]
    gen = torch.Generator(device=dev)
    copies = []
    for c in range(3):
        gen.manual_seed(synthetic.seed_of("bench", "outliers", c) % (2 ** 62))
        W = torch.randn((N, K), generator=gen, device=dev) * 0.02
        mask = torch.rand((N, K), generator=gen, device=dev) < 0.001
        W = torch.where(mask, torch.randn((N, K), generator=gen, device=dev) * synthetic.OUTLIER_STD, W)
        copies.append(w4.w4_quantize_outliers(W))
        del W, mask
    X = torch.randn((1, K), generator=gen, device=dev).to(torch.bfloat16)
    Y = torch.empty((1, N), dtype=torch.float32, device=dev)
    ws = w4.workspace(1, N, K, dev)
    stream = torch.cuda.Stream()
    res = {}
    for name, fn in (("plain", lambda i: w4.w4a16_gemm(X, *copies[i % 3][:3], out=Y, ws=ws)),
                     ("with_outliers", lambda i: w4.w4a16_gemm_outliers(X, *copies[i % 3], out=Y, ws=ws))):
        g = _graph_of(fn, launches, 3, stream)
        res[name] = _replay_timed(g, stream) / launches * 1e3
        del g
    row_ptr, col, val = copies[0][3]
    nbytes = gemm_bytes(1, N, K) + (N + 1) * 4 + col.numel() * 6
    out = {"us_per_call": round(res["with_outliers"], 3), "us_per_call_dense_only": round(res["plain"], 3),
           "GB/s": round(nbytes / (res["with_outliers"] * 1e-6) / 1e9, 1), "nnz": int(col.numel()),
           "workload": "gate_up 4096->28672, M=1, 0.1% of W in fp16 CSR (N(0,0.02) W with 0.1% N(0,0.4) outliers)"}
    del copies
    torch.cuda.empty_cache()
    return out


def gptq_leg(w4):
    """GPTQ column sweep of the Llama-3-8B o_proj weights (4096 x 4096) with a 512-row
    calibration batch (correlated channels): device time per layer (synchronous call)."""
    dev = torch.device("cuda")
    K, N = synthetic.SHAPES_8B["o_proj"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(synthetic.seed_of("bench", "gptq") % (2 ** 62))
    W = torch.randn((N, K), generator=gen, device=dev) * 0.02
    X = torch.randn((512, K), generator=gen, device=dev)
    X = (X + 0.5 * X[:, :1]).to(torch.bfloat16)
    w4.w4_quantize_gptq(W, X)  # warm-up
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    packed, scales, zeros = w4.w4_quantize_gptq(W, X)
    ms = (time.perf_counter() - t0) * 1e3
    Xf = X.float()
    y = Xf @ W.t()
    rtn = w4.w4_quantize(W)
    err = {}
    for name, (p, sc, z) in (("gptq", (packed, scales, zeros)), ("rtn", rtn)):
        err[name] = float(((y - w4.w4a16_gemm(X, p, sc, z)) ** 2).sum())
    out = {"ms_per_layer": round(ms, 1), "output_error_vs_rtn": round(err["gptq"] / err["rtn"], 4),
           "workload": "o_proj 4096x4096 fp32 W, 512 x 4096 bf16 calibration (correlated channels), group 128"}
    del W, X, Xf, y
    torch.cuda.empty_cache()
    return out


def awq_search_leg(w4, repeats=3):
    """AWQ exponent search on the Llama-3-8B gate_up weights with a 512-row calibration batch
    (1% of the channels x10), 21 exponents in [-1, 1]: device time per search."""
    dev = torch.device("cuda")
    K, N = synthetic.SHAPES_8B["gate_up"]
    gen = torch.Generator(device=dev)
    gen.manual_seed(synthetic.seed_of("bench", "awq-search") % (2 ** 62))
    W = torch.randn((N, K), generator=gen, device=dev) * 0.02
    X = torch.randn((512, K), generator=gen, device=dev)
    X[:, torch.randperm(K, generator=gen, device=dev)[: K // 100]] *= 10.0
    X = X.to(torch.bfloat16)
    w4.w4_awq_search(W, X)  # warm-up
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(repeats):
        _, best, errs = w4.w4_awq_search(W, X)
    b.record()
    torch.cuda.synchronize()
    zero = errs[w4.AWQ_EXPONENTS.index(0.0)]
    out = {"ms_per_search": round(a.elapsed_time(b) / repeats, 3), "exponents": len(w4.AWQ_EXPONENTS),
           "best_exponent": best, "error_vs_plain_rtn": round(min(errs) / zero, 4),
           "workload": "gate_up 4096->28672 fp32 W, 512 x 4096 bf16 calibration with 1% channels x10"}
    del W, X
    torch.cuda.empty_cache()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the quantize and prefill legs")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"

    world, rank, local = dist_setup(args.gpus)
    from weight_only_int4_w4_b200 import w4  # fails loudly if libw4.so is missing

    hbm_peak, bf16_peak, bf16_sust, peak_src = peaks()
    layers = build_decode_state(w4, torch.device("cuda"))
    step_bytes = sum(gemm_bytes(1, layers[n]["N"], layers[n]["K"]) for n in LAYERS)

    ms, clocks, repeats = decode_leg(w4, layers, args.steps, args.warmup, world)
    value, ms = job_throughput(step_bytes * args.steps, ms, world)

    K, N = synthetic.SHAPES_8B[DOMINANT]
    dom_bytes = gemm_bytes(1, N, K)
    dom_ms = dominant_leg(w4, layers, max(20, args.steps), args.warmup)
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9

    e2e_ms, h2d, d2h = e2e_leg(w4, layers, max(20, args.steps // 4), args.warmup, world)
    e2e_value, e2e_ms = job_throughput(step_bytes * max(20, args.steps // 4), e2e_ms, world)
    eb_ms, eb_h2d, eb_d2h = e2e_batch_leg(w4, layers, max(20, args.steps // 4), args.warmup, world)
    eb_value, eb_ms = job_throughput(step_bytes * max(20, args.steps // 4), eb_ms, world)
    del layers
    torch.cuda.empty_cache()

    extras = {}
    if not args.no_extras:
        q_ms, q_bytes = quantize_leg(w4)
        q_gbs = q_bytes / (q_ms * 1e-3) / 1e9
        extras["quantize"] = {"value": round(q_gbs, 1), "unit": "GB/s", "ms_per_call_4_layers": round(q_ms, 4),
                              "workload": "quantize+pack of the 4 Llama-3-8B layers, fp32 W",
                              "roofline": {"bound": "hbm", "achieved": round(q_gbs, 1), "peak": hbm_peak,
                                           "unit": "GB/s", "frac": round(q_gbs / hbm_peak, 4),
                                           "frac_nominal": round(q_gbs / NOMINAL_HBM_GBS, 4)}}
        pf = prefill_leg(w4, bf16_peak)
        extras["stack70b"] = stack70b_leg(w4)
        extras["verify_8b"] = verify_leg(w4)
        extras["awq_search"] = awq_search_leg(w4)
        extras["gptq"] = gptq_leg(w4)
        extras["outliers"] = outlier_leg(w4)
        big = pf[f"M{max(PREFILL_MS)}"]
        extras["prefill"] = {"value": big["tflops"], "unit": "TFLOP/s", "ms_per_step": big["ms_per_step"],
                             "workload": "Llama-3-70B qkv/o_proj/gate_up/down, bf16 X, M in {512, 2048, 8192}; "
                                         "value = the four layers at M=8192",
                             "by_M": pf,
                             "roofline": {"bound": "tensor", "achieved": big["tflops"], "peak": bf16_peak,
                                          "unit": "TFLOP/s", "frac": big["frac"],
                                          "frac_nominal": big["frac_nominal"], "peak_nominal": NOMINAL_BF16_TFLOPS}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = time_cpu_oracle()
        extras["cpu_baseline_all_cores"], extras["cpu_baseline_stack70b"] = time_cpu_oracle_all_cores()

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16xu4->f32", "data": "synthetic",
            "config": {**decode_config(world),
                       "l2": f"{N_COPIES} rotating weight copies ({N_COPIES * step_bytes / 1e6:.0f} MB > 4x L2): "
                             "each step reads weights not touched for 4 steps",
                       "graph": "timed steps captured in one CUDA graph"},
            "roofline": {"bound": "hbm", "kernel": f"gemv_mma ({DOMINANT} 4096->28672, M=1)",
                         "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(achieved / hbm_peak, 4), "peak_source": peak_src,
                         "peak_nominal": NOMINAL_HBM_GBS, "frac_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                         "step_frac": round(value / world / hbm_peak, 4),
                         "bytes_per_launch": dom_bytes, "avg_launch_us": round(dom_ms * 1e3, 3),
                         "traffic": committed_traffic("gemv_mma_gate_up_m1")},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "api": "w4a16_gemm_host_async per layer (pinned host X/Y, copies enqueued with the matmul), one stream wait per step",
                    "note": "the gap to value is host-side enqueueing of 4 x (copy in, matmul, copy out) and one "
                            "host synchronization per step; the copies themselves are only h2d+d2h bytes per step"},
            "e2e_batched": {"value": round(eb_value, 2), "unit": "GB/s", "h2d_bytes_per_step": eb_h2d,
                            "d2h_bytes_per_step": eb_d2h,
                            "api": "w4a16_gemm_host_batch_async: the step's four independent matmuls in one call "
                                   "(one copy in, four matmuls, one copy out), one stream wait per step"},
            "gpu_launches": 4 * args.steps,
            "clocks": clocks,
            "repeats": repeats,
            "cpu_baseline": cpu,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
