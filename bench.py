"""Benchmark of the AWQ W4A16 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (`value`): decode GEMV throughput over one Mistral-7B-shaped layer at M=1
(q/k/v/o 4096->4096/1024/1024/4096, gate/up 4096->14336, down 14336->4096), group 128,
zero point on, in GB/s of algorithmic bytes (packed codes + fp16 scales + packed zeros
+ x + y).  One step = one pass over the layer with q/k/v and gate/up fused (their
weights concatenated row-wise: 4 dependent launches, the same bytes), each from a
different copy of the layer's weights so that every step reads HBM (4 rotated copies,
454 MB > 3x L2).  The seven-launch (unfused) number is reported beside it.
The same line also measures the other rows of the path:
  gemm         tcgen05 W4A16 GEMM on Llama-70B-shaped prefill linears at M=2048 (TFLOP/s)
  quantize     awq_quantize_pack on the 4096x4096 layer (GB/s)
  scale_search awq_scale_search on 4096x4096 with 512 calibration tokens, 20 alphas
With --gpus N (torchrun) every rank runs the same work on its own GPU (independent
layers, no data-path collective): weak scaling, value = sum over ranks.
`--impl reference` times the CPU oracle on a bounded sample of the same workload.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import inputs  # noqa: E402

G = 128
ZP = True
ROTATIONS = 4
METRIC = "W4A16 linear: GEMV HBM GB/s (% of peak); GEMM TFLOPS (% of fp16 peak)"
WORKLOAD = "mistral7b-layer-decode-gemv-m1-g128-zp-fused-qkv-gateup"


def packed_bytes(N: int, K: int, g: int = G, zp: bool = ZP) -> int:
    ng = K // g
    return N * K // 2 + N * ng * 2 + (N * ((ng + 7) // 8) * 4 if zp else 0)


def linear_bytes(M: int, N: int, K: int) -> int:
    """Algorithmic bytes of one fused linear: packed weights + x + y."""
    return packed_bytes(N, K) + M * K * 2 + M * N * 2


def layer_bytes(shapes, M=1) -> int:
    return sum(linear_bytes(M, n, k) for _, k, n in shapes)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def profile_traffic(kernel_tag: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or None if the
    summary is missing or was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(gemv_sources())
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel_tag and not line.startswith("#"):
            if parts[2] != digest:
                return None
            return float(parts[1])
    return None


def gemv_sources():
    """The files that define the decode GEMV kernel and its launch configuration: a
    recorded traffic figure stays valid while none of them changes."""
    from bit_weight_only_linear_b200 import build
    names = ("gemv.cuh", "sm100.cuh", "common.cuh", "launch.cuh", "awq_api.cu")
    return [p for p in build.sources() if os.path.basename(p) in names]


def source_digest(paths) -> str:
    """Digest of the code in `paths`: comments and blank lines do not count, so that a
    comment edit does not invalidate a recorded measurement."""
    import hashlib
    import re
    h = hashlib.sha256()
    for p in sorted(paths):
        text = open(p, encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        lines = [re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


class ClockSampler:
    """nvidia-smi SM clock / throttle-reason samples while the timed work runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        rows = []
        for line in open(self.out.name):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9:
                try:
                    rows.append((float(p[1]), float(p[2]), float(p[3]), p[5:9]))
                except ValueError:
                    pass
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, _, r in rows for i, v in enumerate(r) if v.lower() == "active"})
        loaded = [r[0] for r in rows if r[2] > 200.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def _dist_setup(n_gpus, backend="nccl"):
    """Rank / world from the torchrun environment; one process group per job (NCCL on
    the GPUs; the CPU tests use gloo).  Returns (world, rank, local_rank)."""
    import datetime

    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    timeout = datetime.timedelta(seconds=120)
    if world > 1:
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timeout)
    elif backend == "nccl":
        torch.cuda.set_device(0)
    return world, rank, local


def _barrier(world, cuda=True):
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def _max_over_ranks(world, value_ms, device="cuda"):
    """The slowest rank's time: every rank gets the maximum."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return value_ms
    t = torch.tensor([value_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_gbs(world, bytes_per_step, steps, ms):
    """Whole-job throughput: the bytes every rank processed over the slowest rank's
    time (each rank runs its own copy of the work)."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def build_decode_layer(awq, torch, seed_offset, fused=False):
    """Quantise the Mistral linears on the GPU (7, or 4 with q/k/v and gate/up
    concatenated); return per-linear packed tensors (ROTATIONS copies) and inputs."""
    layers = []
    src = (inputs.fused_layer_inputs(1, 0.02, seed_offset) if fused
           else inputs.layer_inputs(inputs.MISTRAL_7B_LAYER, 1, 0.02, seed_offset))
    for name, W, X in src:
        N, K = W.shape
        Wd = torch.from_numpy(W).cuda()
        q, sc, z = awq.quantize_pack(Wd, None, G, ZP)
        copies = [(q, sc, z)] + [(q.clone(), sc.clone(), z.clone()) for _ in range(ROTATIONS - 1)]
        del Wd
        x = torch.from_numpy(X).cuda()
        y = torch.empty((1, N), dtype=torch.float16, device="cuda")
        layers.append(dict(name=name, N=N, K=K, copies=copies, x=x, y=y, x_host=X))
    torch.cuda.synchronize()
    return layers


def time_decode(awq, torch, layers, steps, warmup, world):
    """Main metric: CUDA-graph replay of ROTATIONS layer passes; returns ms per step."""
    stream = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()

    def one_pass(r):
        for L in layers:
            q, sc, z = L["copies"][r]
            awq.linear_gemv(L["x"], q, sc, z, G, ZP, out=L["y"])

    with torch.cuda.stream(stream):
        for r in range(ROTATIONS):       # warm the launch configuration outside capture
            one_pass(r)
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=stream):
        for r in range(ROTATIONS):
            one_pass(r)
    reps = max(1, steps // ROTATIONS)
    steps = reps * ROTATIONS
    for _ in range(max(1, warmup // ROTATIONS + 1)):
        g.replay()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    _barrier(world)
    ms = e0.elapsed_time(e1)
    del g
    return ms, steps


def per_launch_gemv(awq, torch, layers, reps=64):
    """Average device duration of each GEMV launch, for the roofline object: a CUDA
    graph of `reps` launches of one linear (rotating weight copies), timed with CUDA
    events on the stream it is replayed on."""
    out = []
    stream = torch.cuda.Stream()
    for L in layers:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            for r in range(ROTATIONS):
                q, sc, z = L["copies"][r]
                awq.linear_gemv(L["x"], q, sc, z, G, ZP, out=L["y"])
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            for i in range(reps):
                q, sc, z = L["copies"][i % ROTATIONS]
                awq.linear_gemv(L["x"], q, sc, z, G, ZP, out=L["y"])
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(3):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        out.append((L["name"], linear_bytes(1, L["N"], L["K"]), e0.elapsed_time(e1) / (3 * reps)))
        del g
    return out


def time_decode_e2e(awq, torch, layers, steps):
    """Same metric through the C ABI with host buffers: every step copies the layer's
    input vectors host->device (one copy from one pinned buffer), runs the GEMV calls,
    and copies their outputs device->host (one copy into one pinned buffer)."""
    ks = [L["K"] for L in layers]
    ns = [L["N"] for L in layers]
    x_host = torch.from_numpy(np.concatenate([L["x_host"].reshape(-1) for L in layers])).pin_memory()
    y_host = torch.empty(sum(ns), dtype=torch.float16).pin_memory()
    x_dev = torch.empty_like(x_host, device="cuda")
    y_dev = torch.empty(sum(ns), dtype=torch.float16, device="cuda")
    xo = np.cumsum([0] + ks)
    yo = np.cumsum([0] + ns)
    xs = [x_dev[xo[i]:xo[i + 1]].view(1, ks[i]) for i in range(len(layers))]   # 16-byte aligned views
    ys = [y_dev[yo[i]:yo[i + 1]].view(1, ns[i]) for i in range(len(layers))]
    h2d = x_host.numel() * 2
    d2h = y_host.numel() * 2
    s = torch.cuda.current_stream()

    def step(i):
        r = i % ROTATIONS
        x_dev.copy_(x_host, non_blocking=True)
        for L, x, y in zip(layers, xs, ys):
            q, sc, z = L["copies"][r]
            awq.linear_gemv(x, q, sc, z, G, ZP, out=y)
        y_host.copy_(y_dev, non_blocking=True)

    for i in range(8):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(steps):
        step(i)
    e1.record(s)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1), h2d, d2h


def measure_gemm(awq, torch, reps=5):
    """Llama-70B-shaped prefill linears at M=2048 through awq_linear_gemm (TFLOP/s)."""
    tot_flop, tot_ms, per = 0.0, 0.0, []
    for i, (name, K, N) in enumerate(inputs.LLAMA_70B_FUSED):
        W = torch.from_numpy(inputs.weights(N, K, 0.015, inputs.SEED_W + 30 + i)).cuda()
        q, sc, z = awq.quantize_pack(W, None, G, ZP)
        del W
        X = torch.from_numpy(inputs.activations(2048, K, inputs.SEED_X + 30 + i, inputs.SEED_OUTLIER + 30)).cuda()
        Y = torch.empty((2048, N), dtype=torch.float16, device="cuda")
        try:
            awq.linear_gemm(X, q, sc, z, G, ZP, out=Y)
        except awq.AWQError as e:
            return {"unavailable": str(e)}
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            awq.linear_gemm(X, q, sc, z, G, ZP, out=Y)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / reps
        flop = 2.0 * 2048 * N * K
        per.append({"linear": name, "K": K, "N": N, "us": round(ms * 1e3, 1),
                    "tflops": round(flop / ms / 1e9, 1)})
        tot_flop += flop
        tot_ms += ms
        del q, sc, z, X, Y
    return {"workload": "llama70b-prefill-m2048-g128-zp", "value": round(tot_flop / tot_ms / 1e9, 1),
            "unit": "TFLOP/s", "us_per_layer": round(tot_ms * 1e3, 1), "per_linear": per}


def measure_quantize(awq, torch, reps=20):
    """Device time of the 4096^2 quantise/pack: a CUDA graph of `reps` calls over 10
    rotated weight copies (10 x 32 MiB > 2x L2), timed with events on its stream (a graph,
    so that host call overhead is not what is measured)."""
    W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W)).cuda()
    copies = [W] + [W.clone() for _ in range(9)]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        outs = awq.quantize_pack(W, None, G, ZP)
        for i in range(10):
            awq.quantize_pack(copies[i], None, G, ZP, out=outs)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(reps):
            awq.quantize_pack(copies[i % 10], None, G, ZP, out=outs)
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(3):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (3 * reps)
    del g
    nbytes = 4096 * 4096 * 2 + packed_bytes(4096, 4096)
    return {"workload": "quantize-pack-4096x4096-g128-zp", "value": round(nbytes / ms / 1e6, 1),
            "unit": "GB/s", "us": round(ms * 1e3, 2)}


def measure_search(awq, torch, reps=3):
    W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W + 40)).cuda()
    X = torch.from_numpy(inputs.activations(512, 4096, inputs.SEED_X + 40, inputs.SEED_OUTLIER + 40)).cuda()
    try:
        ws = torch.empty(awq.workspace_bytes(awq.AWQ_OP_SCALE_SEARCH, 512, 4096, 4096, G, ZP),
                         dtype=torch.uint8, device="cuda")
        awq.scale_search(X, W, G, ZP, 20, workspace=ws)
    except awq.AWQError as e:
        return {"unavailable": str(e)}
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        awq.scale_search(X, W, G, ZP, 20, workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    flop = 20 * 2.0 * 512 * 4096 * 4096
    return {"workload": "scale-search-4096x4096-t512-a20-g128-zp", "value": round(flop / ms / 1e9, 1),
            "unit": "TFLOP/s", "ms": round(ms, 3)}


def cpu_baseline_sample(seconds: float = 12.0):
    """The oracle, as it stands, on a bounded sample of the decode workload: the first
    256 output channels of each of the four fused linears (fp64 dequantise + matmul)."""
    from oracle import awq_oracle as O
    sample = []
    for name, W, X in inputs.fused_layer_inputs(1, 0.02):
        Ws = W[:256]
        q, sc, z = O.quantize_pack(Ws, None, G, ZP)
        sample.append((X, q, sc, z, W.shape[1]))
    nbytes = sum(linear_bytes(1, 256, k) for *_, k in sample)
    t0 = time.perf_counter()
    passes = 0
    while True:
        for X, q, sc, z, K in sample:
            O.linear(X, q, sc, z, K, G, ZP)
        passes += 1
        if time.perf_counter() - t0 > seconds:
            break
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    return {"value": round(nbytes * passes / dt / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"first 256 output channels of each of the 4 fused linears ({nbytes} algorithmic bytes per "
                      f"pass), {passes} passes in {dt:.1f} s"}


def run_ours(args):
    import torch
    from bit_weight_only_linear_b200 import awq, build
    world, rank, local = _dist_setup(args.gpus)
    if rank == 0:
        build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    awq.load_library()
    peaks = read_peaks()
    # the seven linears as separate launches (reported beside the headline)
    unfused = build_decode_layer(awq, torch, seed_offset=rank * 100, fused=False)
    step_bytes_7 = layer_bytes(inputs.MISTRAL_7B_LAYER, 1)
    ms7, steps7 = time_decode(awq, torch, unfused, args.steps, args.warmup, world)
    ms7 = _max_over_ranks(world, ms7)
    launches7 = per_launch_gemv(awq, torch, unfused)
    for L in unfused:
        L.clear()
    del unfused
    torch.cuda.empty_cache()

    # headline: the layer with q/k/v and gate/up fused (4 dependent launches per step)
    layers = build_decode_layer(awq, torch, seed_offset=rank * 100, fused=True)
    step_bytes = sum(linear_bytes(1, n, k) for _, k, n, _ in inputs.MISTRAL_7B_LAYER_FUSED)

    with ClockSampler(local) as clocks:
        ms, steps = time_decode(awq, torch, layers, args.steps, args.warmup, world)
    ms = _max_over_ranks(world, ms)
    clk = clocks.summary()
    value = aggregate_gbs(world, step_bytes, steps, ms)

    launches = per_launch_gemv(awq, torch, layers)
    kern_bytes = sum(b for _, b, _ in launches)
    kern_ms = sum(t for _, _, t in launches)
    achieved = kern_bytes / (kern_ms * 1e-3) / 1e9
    traffic = profile_traffic("gemv_mistral7b_layer")
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                "peak_source": peaks["source"] + " (burst copy bandwidth)",
                "per_linear_us": {n: round(t * 1e3, 2) for n, _, t in launches}}
    unfused_obj = {"workload": "mistral7b-layer-decode-gemv-m1-g128-zp-unfused",
                   "value": round(aggregate_gbs(world, step_bytes_7, steps7, ms7), 1), "unit": "GB/s",
                   "ms_per_step": round(ms7 / steps7, 5), "launches_per_step": 7,
                   "per_linear_us": {n: round(t * 1e3, 2) for n, _, t in launches7}}

    e2e_steps = max(50, min(args.steps, 400))
    # note: time_decode_e2e copies each fused linear's input once per step
    e2e_ms, h2d, d2h = time_decode_e2e(awq, torch, layers, e2e_steps)
    e2e_ms = _max_over_ranks(world, e2e_ms)
    e2e = {"value": round(aggregate_gbs(world, step_bytes, e2e_steps, e2e_ms), 1), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    for L in layers:
        L.clear()
    torch.cuda.empty_cache()
    extra = {}
    if not args.skip_extra:
        extra["gemm"] = measure_gemm(awq, torch)
        if "value" in extra["gemm"]:
            extra["gemm"]["frac"] = round(extra["gemm"]["value"] / peaks["bf16_tflops"], 4)
            extra["gemm"]["peak"] = peaks["bf16_tflops"]
        extra["quantize"] = measure_quantize(awq, torch)
        extra["scale_search"] = measure_search(awq, torch)

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        cpu = cpu_baseline_sample()

    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
                "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms / steps, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u4-f16-f32acc",
                "data": "synthetic (seeded fp16 N(0,0.02^2) weights, N(0,1) activations with 1% x20 channels)",
                "config": {"workload": WORKLOAD,
                           "linears": [f"{n}:{k}->{nn}" for n, k, nn, _ in inputs.MISTRAL_7B_LAYER_FUSED],
                           "fusion": "q/k/v and gate/up weights concatenated row-wise (layer fusion); "
                                     "same bytes as the seven linears",
                           "batch_m": 1, "group_size": G, "zero_point": ZP, "bytes_per_step": step_bytes,
                           "l2": f"weights rotated over {ROTATIONS} copies ({ROTATIONS * step_bytes / 1e6:.0f} MB > 3x L2)",
                           "timing": "CUDA graph of 4 layer passes, CUDA events, max over ranks"},
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": len(inputs.MISTRAL_7B_LAYER_FUSED) * steps, "clocks": clk,
                "unfused": unfused_obj, **extra}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_reference(args):
    """The oracle as it stands on the host cores: each step is a bounded sample of the
    decode workload (up to 256 output channels of each of the 4 fused linears)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import awq_oracle as O
    layer = list(inputs.fused_layer_inputs(1, 0.02))

    def make_sample(rows):
        out = []
        for name, W, X in layer:
            q, sc, z = O.quantize_pack(W[:rows], None, G, ZP)
            out.append((X, q, sc, z, W.shape[1]))
        return out

    def step():
        for X, q, sc, z, K in sample:
            O.linear(X, q, sc, z, K, G, ZP)

    # size the per-step sample so that the whole run stays within about two minutes
    rows = 256
    sample = make_sample(rows)
    t0 = time.perf_counter()
    step()
    t_step = time.perf_counter() - t0
    budget = 100.0 / max(1, args.steps + args.warmup)
    if t_step > budget:
        rows = max(8, int(rows * budget / t_step) // 8 * 8)
        sample = make_sample(rows)
    nbytes = sum(linear_bytes(1, rows, k) for *_, k in sample)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    value = nbytes * args.steps / dt / 1e9
    sample_desc = f"first {rows} output channels of each of the 4 fused Mistral-7B linears per step"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample_desc},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample_desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile(args):
    """Profiling mode (no timing, no JSON): quantise the fused decode layer once, run
    one warm-up pass and one pass of its four GEMV launches, run one launch of each
    of the four Llama-70B prefill GEMMs, and exit.  ncu captures select kernels from
    this with -k / -s / -c."""
    import torch
    from bit_weight_only_linear_b200 import awq, build
    build.build()
    awq.load_library()
    torch.cuda.set_device(0)
    layers = build_decode_layer(awq, torch, 0, fused=True)
    for _ in range(2):
        for L in layers:
            q, sc, z = L["copies"][0]
            awq.linear_gemv(L["x"], q, sc, z, G, ZP, out=L["y"])
    torch.cuda.synchronize()
    for L in layers:
        L.clear()
    torch.cuda.empty_cache()
    if not args.skip_extra:
        for i, (name, K, N) in enumerate(inputs.LLAMA_70B_FUSED):
            W = torch.from_numpy(inputs.weights(N, K, 0.015, inputs.SEED_W + 30 + i)).cuda()
            q, sc, z = awq.quantize_pack(W, None, G, ZP)
            del W
            X = torch.from_numpy(inputs.activations(2048, K, inputs.SEED_X + 30 + i, inputs.SEED_OUTLIER + 30)).cuda()
            awq.linear_gemm(X, q, sc, z, G, ZP)
            torch.cuda.synchronize()
            del q, sc, z, X
    awq.device_error()
    print("profile run done", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-extra", action="store_true", help="headline decode measurement only")
    ap.add_argument("--skip-cpu", action="store_true", help="do not time the CPU oracle")
    ap.add_argument("--profile", action="store_true",
                    help="no timing: one pass of the decode layer and one launch of each prefill GEMM, for ncu")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile:
        run_profile(args)
        return
    if args.impl == "reference":
        if args.steps == 2000:
            args.steps = 20
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
