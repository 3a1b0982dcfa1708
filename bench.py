"""Benchmark of the AWQ W4A16 hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Headline (`value`): decode GEMV throughput over one Mistral-7B-shaped layer at M=1
(q/k/v/o 4096->4096/1024/1024/4096, gate/up 4096->14336, down 14336->4096), group 128,
zero point on, in GB/s of algorithmic bytes (packed codes + fp16 scales + packed zeros
+ x + y).  One step = one pass over the layer with q/k/v and gate/up fused (their
weights concatenated row-wise: 4 dependent launches, the same bytes), each step from a
different copy of the layer's weights so that every step reads HBM (4 rotated copies,
454 MB > 3x L2).  K steps are timed per trial (CUDA graph replays, CUDA events on the
replay stream); the reported time is the median of the trials.

The same JSON line measures every other workload of the path:
  single_gemv   one 4096x4096 GEMV at M=1 (32 rotated weight copies, > 2x L2)
  unfused       the seven Mistral-7B linears as seven launches
  batched       the seven linears at M in {1, 4, 8, 16, 64}: GEMV (M <= 8) and GEMM per
                layer, and the measured GEMV -> GEMM crossover
  gemm          tcgen05 W4A16 GEMM on Llama-70B-shaped prefill linears at M=2048
  quantize      awq_quantize_pack on the 4096x4096 layer (GB/s)
  scale_search  awq_scale_search on 4096x4096 with 512 calibration tokens, 20 alphas
  sweep         per group size {32,64,128,256} x zero point {on,off} on that layer:
                search, quantise/pack with s*, GEMV at M=1 and GEMM at M=512 on X'
With --gpus N (torchrun) every rank runs the same work on its own GPU (independent
layers, no data-path collective): weak scaling, value = sum over ranks.
`--impl reference` times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
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
TRIALS = 7
METRIC = "W4A16 linear: GEMV HBM GB/s (% of peak); GEMM TFLOPS (% of fp16 peak)"
WORKLOAD = "mistral7b-layer-decode-gemv-m1-g128-zp-fused-qkv-gateup"
L2_BYTES = 126 * 1024 * 1024
# nominal datasheet peaks (context beside the measured ones)
SPEC_HBM_GBS = 7700.0
SPEC_FP16_TFLOPS = 2250.0
BATCHED_M = (1, 4, 8, 16, 64)
BATCHED_SEED_OFFSET = 20
SWEEP_SEED_OFFSET = 40


def packed_bytes(N: int, K: int, g: int = G, zp: bool = ZP) -> int:
    ng = K // g
    return N * K // 2 + N * ng * 2 + (N * ((ng + 7) // 8) * 4 if zp else 0)


def linear_bytes(M: int, N: int, K: int, g: int = G, zp: bool = ZP) -> int:
    """Algorithmic bytes of one linear: packed weights + x + y."""
    return packed_bytes(N, K, g, zp) + M * K * 2 + M * N * 2


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


# ---------------------------------------------------------------------------
# recorded DRAM traffic (profiles/traffic.txt), valid only for the code it was taken on
# ---------------------------------------------------------------------------

KERNEL_SOURCES = {
    # tag: the files whose code defines the kernel and its launch configuration
    "gemv_mistral7b_layer": ("gemv.cuh", "gemv_launch.cuh", "sm100.cuh", "common.cuh", "launch.cuh"),
    "gemm_llama70b_o_proj": ("gemm_sm100.cuh", "sm100.cuh", "common.cuh"),
    "quantize_pack_4096": ("quantize.cuh", "common.cuh"),
    "search_fused_4096": ("search.cuh", "quantize.cuh", "gemm_sm100.cuh", "sm100.cuh", "common.cuh"),
    "apply_clip_4096": ("clip.cuh", "search.cuh", "quantize.cuh", "gemm_sm100.cuh", "sm100.cuh", "common.cuh"),
}


def kernel_sources(tag: str):
    from bit_weight_only_linear_b200 import build
    names = KERNEL_SOURCES[tag]
    return [p for p in build.sources() if os.path.basename(p) in names]


def gemv_sources():
    return kernel_sources("gemv_mistral7b_layer")


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


def profile_traffic(kernel_tag: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, or None if the
    summary is missing or was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path) or kernel_tag not in KERNEL_SOURCES:
        return None
    digest = source_digest(kernel_sources(kernel_tag))
    for line in open(path):
        parts = line.split()
        if len(parts) >= 3 and parts[0] == kernel_tag and not line.startswith("#"):
            if parts[2] != digest:
                return None
            return float(parts[1])
    return None


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
# process group plumbing (NCCL on the GPUs; the CPU tests use gloo)
# ---------------------------------------------------------------------------

def _dist_setup(n_gpus, backend="nccl"):
    """Rank / world from the torchrun environment; one process group per job.
    Returns (world, rank, local_rank)."""
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


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------

def graph_trials(torch, body, reps, trials=TRIALS, stream=None):
    """Capture body() (a sequence of library calls on the current stream) into a CUDA
    graph on a side stream after one eager warm-up call, replay it once more untimed,
    then time `trials` trials of `reps` replays each with CUDA events recorded on the
    replay stream.  Returns the per-replay milliseconds of each trial."""
    stream = stream or torch.cuda.Stream()
    with torch.cuda.stream(stream):
        body()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        body()
    g.replay()
    torch.cuda.synchronize()
    out = []
    for _ in range(trials):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) / reps)
    del g
    return out


def med(xs):
    return statistics.median(xs)


def rotations_for(nbytes: int, floor: int = 2) -> int:
    """Copies of a working set so that a pass over them all exceeds twice the L2."""
    return max(floor, -(-2 * L2_BYTES // max(1, nbytes)) + 1)


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def build_decode_layer(awq, torch, seed_offset, fused=False, M=1, rotations=ROTATIONS, shapes=None):
    """Quantise the Mistral linears on the GPU (7, or 4 with q/k/v and gate/up
    concatenated); return per-linear packed tensors (`rotations` copies) and inputs."""
    layers = []
    if shapes is not None:
        src = inputs.layer_inputs(shapes, M, 0.02, seed_offset)
    elif fused:
        src = inputs.fused_layer_inputs(M, 0.02, seed_offset)
    else:
        src = inputs.layer_inputs(inputs.MISTRAL_7B_LAYER, M, 0.02, seed_offset)
    for name, W, X in src:
        N, K = W.shape
        Wd = torch.from_numpy(W).cuda()
        q, sc, z = awq.quantize_pack(Wd, None, G, ZP)
        copies = [(q, sc, z)] + [(q.clone(), sc.clone(), z.clone()) for _ in range(rotations - 1)]
        del Wd
        x = torch.from_numpy(X).cuda()
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        layers.append(dict(name=name, N=N, K=K, copies=copies, x=x, y=y, x_host=X))
    torch.cuda.synchronize()
    return layers


def time_decode(awq, torch, layers, steps, world):
    """Headline timing: a CUDA graph of ROTATIONS layer passes (one pass = one step), K
    steps per trial; returns (ms for K steps of each trial, K)."""
    reps = max(1, steps // ROTATIONS)
    steps = reps * ROTATIONS

    def body():
        for r in range(ROTATIONS):
            for L in layers:
                q, sc, z = L["copies"][r]
                awq.linear_gemv(L["x"], q, sc, z, G, ZP, out=L["y"])

    _barrier(world)
    per_replay = graph_trials(torch, body, reps)
    _barrier(world)
    return [t * reps for t in per_replay], steps


def per_launch_gemv(awq, torch, layers, reps=64):
    """Median device duration of each GEMV launch (graph of `reps` launches of one linear
    over its rotating weight copies, events on the replay stream)."""
    out = []
    for L in layers:
        def body(L=L):
            for i in range(reps):
                q, sc, z = L["copies"][i % len(L["copies"])]
                awq.linear_gemv(L["x"], q, sc, z, G, ZP, out=L["y"])
        t = med(graph_trials(torch, body, 3, trials=5)) / reps
        out.append((L["name"], linear_bytes(L["x"].shape[0], L["N"], L["K"]), t))
    return out


def time_decode_e2e(awq, torch, layers, steps):
    """The headline metric through the C ABI with host buffers: every step copies the
    layer's input vectors host->device (one copy from one pinned buffer), makes the four
    GEMV calls and copies their outputs device->host (one copy into one pinned buffer).
    Returns (eager ms, graph ms, h2d bytes, d2h bytes): `eager` issues the calls one by
    one from Python each step; `graph` replays one CUDA graph per step holding the same
    copies and calls."""
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

    def step(r):
        x_dev.copy_(x_host, non_blocking=True)
        for L, x, y in zip(layers, xs, ys):
            q, sc, z = L["copies"][r]
            awq.linear_gemv(x, q, sc, z, G, ZP, out=y)
        y_host.copy_(y_dev, non_blocking=True)

    s = torch.cuda.current_stream()
    for i in range(8):
        step(i % ROTATIONS)
    torch.cuda.synchronize()
    eager = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for i in range(steps):
            step(i % ROTATIONS)
        e1.record(s)
        torch.cuda.synchronize()
        eager.append(e0.elapsed_time(e1))
    # one graph per rotation, replayed in turn: one launch per step from the host
    stream = torch.cuda.Stream()
    graphs = []
    for r in range(ROTATIONS):
        with torch.cuda.stream(stream):
            step(r)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(r)
        graphs.append(g)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    graphed = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(steps):
                graphs[i % ROTATIONS].replay()
            e1.record(stream)
        torch.cuda.synchronize()
        graphed.append(e0.elapsed_time(e1))
    del graphs
    return med(eager), med(graphed), h2d, d2h


def time_decode_e2e_pipelined(awq, torch, layers, steps, per_graph=8, depth=2):
    """The same end-to-end step with its copies overlapped across steps: step i's inputs
    go host->device on an upload stream while step i-1's GEMVs run, and its outputs come
    back device->host on a download stream while step i+1's GEMVs run.  Every step still
    copies its own inputs from pinned memory and reads its own outputs into pinned
    memory; `depth` device/host buffer pairs carry the steps in flight, and events order
    each buffer's reuse.  Returns (eager ms, graph ms) for `steps` steps: `eager` issues
    every call from Python; `graph` replays a captured run of `per_graph` steps (one
    replay covers every weight rotation twice; the pipeline fills and drains once per
    replay)."""
    ks = [L["K"] for L in layers]
    ns = [L["N"] for L in layers]
    xo = np.cumsum([0] + ks)
    yo = np.cumsum([0] + ns)
    x_np = np.concatenate([L["x_host"].reshape(-1) for L in layers])
    x_host = [torch.from_numpy(x_np.copy()).pin_memory() for _ in range(depth)]
    y_host = [torch.empty(sum(ns), dtype=torch.float16).pin_memory() for _ in range(depth)]
    x_dev = [torch.empty(x_np.size, dtype=torch.float16, device="cuda") for _ in range(depth)]
    y_dev = [torch.empty(sum(ns), dtype=torch.float16, device="cuda") for _ in range(depth)]
    xs = [[x[xo[i]:xo[i + 1]].view(1, ks[i]) for i in range(len(layers))] for x in x_dev]
    ys = [[y[yo[i]:yo[i + 1]].view(1, ns[i]) for i in range(len(layers))] for y in y_dev]
    comp, up, down = torch.cuda.current_stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def run(n, start):
        """Issue steps start .. start+n-1 on the three streams (inside a capture too)."""
        ev = {k: [torch.cuda.Event() for _ in range(depth)] for k in ("up", "comp", "down")}
        seen = {k: [False] * depth for k in ev}
        fork = torch.cuda.Event()
        fork.record(comp)
        up.wait_event(fork)
        down.wait_event(fork)
        for i in range(start, start + n):
            b, r = i % depth, i % ROTATIONS
            with torch.cuda.stream(up):
                if seen["comp"][b]:
                    up.wait_event(ev["comp"][b])          # the GEMVs that read x_dev[b] are done
                x_dev[b].copy_(x_host[b], non_blocking=True)
                ev["up"][b].record(up)
                seen["up"][b] = True
            with torch.cuda.stream(comp):
                comp.wait_event(ev["up"][b])
                if seen["down"][b]:
                    comp.wait_event(ev["down"][b])        # y_dev[b] has been read back
                for L, x, y in zip(layers, xs[b], ys[b]):
                    q, sc, z = L["copies"][r]
                    awq.linear_gemv(x, q, sc, z, G, ZP, out=y)
                ev["comp"][b].record(comp)
                seen["comp"][b] = True
            with torch.cuda.stream(down):
                down.wait_event(ev["comp"][b])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                ev["down"][b].record(down)
                seen["down"][b] = True
        comp.wait_stream(up)
        comp.wait_stream(down)

    run(8, 0)
    torch.cuda.synchronize()
    eager = []
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        run(steps, 0)
        e1.record(comp)
        torch.cuda.synchronize()
        eager.append(e0.elapsed_time(e1))
    gstream = torch.cuda.Stream()
    with torch.cuda.stream(gstream):
        comp = gstream
        run(per_graph, 0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gstream):
            run(per_graph, 0)
        g.replay()
        torch.cuda.synchronize()
        reps = max(1, -(-steps // per_graph))
        graphed = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(gstream)
            for _ in range(reps):
                g.replay()
            e1.record(gstream)
            torch.cuda.synchronize()
            graphed.append(e0.elapsed_time(e1) * steps / (reps * per_graph))
        del g
    return med(eager), med(graphed)


def measure_single_gemv(awq, torch, peaks):
    """One 4096x4096 GEMV at M=1 (G=128, zero point): 32 rotated weight copies."""
    K = N = 4096
    W = torch.from_numpy(inputs.weights(N, K, 0.02, inputs.SEED_W)).cuda()
    x = torch.from_numpy(inputs.activations(1, K, inputs.SEED_X)).cuda()
    q, sc, z = awq.quantize_pack(W, None, G, ZP)
    nb = linear_bytes(1, N, K)
    rot = rotations_for(nb)
    copies = [(q, sc, z)] + [(q.clone(), sc.clone(), z.clone()) for _ in range(rot - 1)]
    y = torch.empty((1, N), dtype=torch.float16, device="cuda")
    reps = 4 * rot

    def body():
        for i in range(reps):
            awq.linear_gemv(x, *copies[i % rot], G, ZP, out=y)
    ts = [t / reps for t in graph_trials(torch, body, 2)]
    us = med(ts) * 1e3
    gbs = nb / (us * 1e-6) / 1e9
    return {"workload": "gemv-4096x4096-m1-g128-zp", "value": round(gbs, 1), "unit": "GB/s", "us": round(us, 3),
            "frac": round(gbs / peaks["hbm_gbs"], 4), "frac_spec": round(gbs / SPEC_HBM_GBS, 4),
            "bytes": nb, "l2": f"{rot} rotated weight copies ({rot * nb / 1e6:.0f} MB)",
            "timing": f"median of {TRIALS} trials, CUDA graph of {reps} launches"}


def measure_batched(awq, torch, peaks):
    """The seven Mistral-7B linears at M in BATCHED_M: GEMV (M <= 8) and GEMM per layer."""
    out = {"workload": "mistral7b-layer-batched-decode-g128-zp", "per_m": [], "unit_layer": "us"}
    shapes = inputs.MISTRAL_7B_LAYER
    layers = None
    for M in BATCHED_M:
        if layers is not None:
            for L in layers:
                L.clear()
        torch.cuda.empty_cache()
        layers = build_decode_layer(awq, torch, BATCHED_SEED_OFFSET, M=M, rotations=3, shapes=shapes)
        nb = sum(linear_bytes(M, L["N"], L["K"]) for L in layers)
        flop = sum(2.0 * M * L["N"] * L["K"] for L in layers)
        row = {"M": M, "bytes": nb, "flop": flop}
        for kind in (("gemv", "gemm") if M <= 8 else ("gemm",)):
            fn = awq.linear_gemv if kind == "gemv" else awq.linear_gemm

            def body(fn=fn):
                for r in range(3):
                    for L in layers:
                        fn(L["x"], *L["copies"][r], G, ZP, out=L["y"])
            us = med(graph_trials(torch, body, 4)) / 3 * 1e3
            row[kind] = {"us_per_layer": round(us, 2), "gbs": round(nb / (us * 1e-6) / 1e9, 1),
                         "tflops": round(flop / (us * 1e-6) / 1e12, 2),
                         "frac_hbm": round(nb / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 4)}
        out["per_m"].append(row)
    for L in layers:
        L.clear()
    torch.cuda.empty_cache()
    faster = [r["M"] for r in out["per_m"] if "gemv" in r and r["gemm"]["us_per_layer"] < r["gemv"]["us_per_layer"]]
    out["crossover"] = ("GEMM faster from M=%d" % min(faster)) if faster else \
        "GEMV faster at every M <= 8 it accepts; GEMM for M > 8"
    return out


def measure_gemm(awq, torch, peaks, reps=3):
    """Llama-70B-shaped prefill linears at M=2048 through awq_linear_gemm (TFLOP/s).  Each
    linear rotates over copies of (X, weights) so that every call reads them from HBM."""
    tot_flop, tot_ms, per = 0.0, 0.0, []
    for i, (name, K, N) in enumerate(inputs.LLAMA_70B_FUSED):
        W = torch.from_numpy(inputs.weights(N, K, 0.015, inputs.SEED_W + 30 + i)).cuda()
        q, sc, z = awq.quantize_pack(W, None, G, ZP)
        del W
        X = torch.from_numpy(inputs.activations(2048, K, inputs.SEED_X + 30 + i, inputs.SEED_OUTLIER + 30)).cuda()
        rot = rotations_for(packed_bytes(N, K) + X.numel() * 2)
        sets = [(X, q, sc, z)] + [(X.clone(), q.clone(), sc.clone(), z.clone()) for _ in range(rot - 1)]
        Y = torch.empty((2048, N), dtype=torch.float16, device="cuda")
        try:
            awq.linear_gemm(X, q, sc, z, G, ZP, out=Y)
        except awq.AWQError as e:
            return {"unavailable": str(e)}

        def body():
            for j in range(rot):
                Xj, qj, scj, zj = sets[j]
                awq.linear_gemm(Xj, qj, scj, zj, G, ZP, out=Y)
        ms = med(graph_trials(torch, body, reps)) / rot
        flop = 2.0 * 2048 * N * K
        per.append({"linear": name, "K": K, "N": N, "us": round(ms * 1e3, 1),
                    "tflops": round(flop / ms / 1e9, 1)})
        tot_flop += flop
        tot_ms += ms
        del sets, q, sc, z, X, Y
        torch.cuda.empty_cache()
    awq.device_error()
    tf = tot_flop / tot_ms / 1e9
    return {"workload": "llama70b-prefill-m2048-g128-zp", "value": round(tf, 1), "unit": "TFLOP/s",
            "us_per_layer": round(tot_ms * 1e3, 1), "per_linear": per,
            "frac": round(tf / peaks["bf16_tflops"], 4), "peak": peaks["bf16_tflops"],
            "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
            "frac_spec": round(tf / SPEC_FP16_TFLOPS, 4),
            "l2": "(X, weights) rotated over copies > 2x L2 per linear",
            "timing": f"median of {TRIALS} trials of CUDA-graph replays"}


def measure_quantize(awq, torch, peaks, G_=G, zp=ZP, W=None, s=None):
    """Device time of the 4096^2 quantise/pack over 10 rotated weight copies (10 x 32 MiB
    > 2x L2), median of trials of CUDA-graph replays."""
    if W is None:
        W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W)).cuda()
    copies = [W] + [W.clone() for _ in range(9)]
    outs = awq.quantize_pack(W, s, G_, zp)

    def body():
        for i in range(10):
            awq.quantize_pack(copies[i], s, G_, zp, out=outs)
    ms = med(graph_trials(torch, body, 3)) / 10
    nbytes = 4096 * 4096 * 2 + packed_bytes(4096, 4096, G_, zp)
    gbs = nbytes / ms / 1e6
    return {"workload": f"quantize-pack-4096x4096-g{G_}-{'zp' if zp else 'sym'}", "value": round(gbs, 1),
            "unit": "GB/s", "us": round(ms * 1e3, 2), "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": nbytes}


def measure_search(awq, torch, peaks, G_=G, zp=ZP, X=None, W=None, reps=3, duo=False):
    if W is None:
        W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W + SWEEP_SEED_OFFSET)).cuda()
        X = torch.from_numpy(inputs.activations(512, 4096, inputs.SEED_X + SWEEP_SEED_OFFSET,
                                                inputs.SEED_OUTLIER + SWEEP_SEED_OFFSET)).cuda()
    try:
        ws = torch.empty(max(16, awq.workspace_bytes(awq.AWQ_OP_SCALE_SEARCH, 512, 4096, 4096, G_, zp)),
                         dtype=torch.uint8, device="cuda")
        res = awq.scale_search(X, W, G_, zp, 20, workspace=ws, duo_scaling=duo)
    except awq.AWQError as e:
        return {"unavailable": str(e)}, None
    s_out, losses, best = res

    def body():
        awq.scale_search(X, W, G_, zp, 20, workspace=ws, out=res, duo_scaling=duo)
    ms = med(graph_trials(torch, body, reps))
    flop = 20 * 2.0 * 512 * 4096 * 4096
    tf = flop / ms / 1e9
    kind = "scale-search-duo" if duo else "scale-search"
    return ({"workload": f"{kind}-4096x4096-t512-a20-g{G_}-{'zp' if zp else 'sym'}",
             "value": round(tf, 1), "unit": "TFLOP/s", "ms": round(ms, 3),
             "frac": round(tf / peaks["bf16_tflops"], 4), "best_index": int(best.item())}, s_out)


def measure_clip(awq, torch, peaks, reps=3, n_clip=10):
    """awq_apply_clip on the 4096x4096 layer with 512 calibration tokens at a searched
    scale (G=128, zero point, 10 ratios): TFLOP/s of the algorithmic 2 M N K n_clip."""
    W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W + SWEEP_SEED_OFFSET)).cuda()
    X = torch.from_numpy(inputs.activations(512, 4096, inputs.SEED_X + SWEEP_SEED_OFFSET,
                                            inputs.SEED_OUTLIER + SWEEP_SEED_OFFSET)).cuda()
    try:
        s, _, _ = awq.scale_search(X, W, G, ZP, 20)
        outs = awq.apply_clip(X, W, s, G, ZP, 20, n_clip)
        need = int(awq.load_library().awq_apply_clip_workspace_bytes(512, 4096, 4096, awq.config(G, ZP), n_clip))
        ws = torch.empty(max(16, need), dtype=torch.uint8, device="cuda")
    except awq.AWQError as e:
        return {"unavailable": str(e)}

    def body():
        awq.apply_clip(X, W, s, G, ZP, 20, n_clip, out=outs, workspace=ws)
    ms = med(graph_trials(torch, body, reps))
    awq.device_error()
    flop = 2.0 * 512 * 4096 * 4096 * n_clip
    tf = flop / ms / 1e9
    return {"workload": f"apply-clip-4096x4096-t512-r{n_clip}-g{G}-zp", "value": round(tf, 1), "unit": "TFLOP/s",
            "ms": round(ms, 3), "frac": round(tf / peaks["bf16_tflops"], 4),
            "clipped_groups": int((outs[3] > 0).sum().item()), "groups": int(outs[3].numel())}


def measure_sweep(awq, torch, peaks):
    """The quantisation sweep on one 4096x4096 layer (512 calibration tokens): per
    (group size, zero point) the search, quantise/pack with s*, then GEMV at M=1 and GEMM
    at M=512 on X' = X / s*."""
    W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W + SWEEP_SEED_OFFSET)).cuda()
    X = torch.from_numpy(inputs.activations(512, 4096, inputs.SEED_X + SWEEP_SEED_OFFSET,
                                            inputs.SEED_OUTLIER + SWEEP_SEED_OFFSET)).cuda()
    rows = []
    for g_ in inputs_group_sizes():
        for zp in (True, False):
            srch, s = measure_search(awq, torch, peaks, g_, zp, X, W)
            if s is None:
                rows.append({"G": g_, "zero_point": zp, **srch})
                continue
            qnt = measure_quantize(awq, torch, peaks, g_, zp, W, s)
            q, sc, z = awq.quantize_pack(W, s, g_, zp)
            Xp = awq.fold_inverse_scale(X, s)
            nb1 = linear_bytes(1, 4096, 4096, g_, zp)
            rot = rotations_for(nb1)
            copies = [(q, sc, z)] + [(q.clone(), sc.clone(), None if z is None else z.clone())
                                     for _ in range(rot - 1)]
            x1 = Xp[:1].contiguous()
            y1 = torch.empty((1, 4096), dtype=torch.float16, device="cuda")

            def gemv_body():
                for i in range(rot):
                    awq.linear_gemv(x1, *copies[i], g_, zp, out=y1)
            us1 = med(graph_trials(torch, gemv_body, 2)) / rot * 1e3
            y2 = torch.empty((512, 4096), dtype=torch.float16, device="cuda")
            xs = [Xp] + [Xp.clone() for _ in range(min(rot, 8) - 1)]

            def gemm_body():
                for i in range(len(xs)):
                    awq.linear_gemm(xs[i], *copies[i], g_, zp, out=y2)
            us2 = med(graph_trials(torch, gemm_body, 2)) / len(xs) * 1e3
            flop2 = 2.0 * 512 * 4096 * 4096
            rows.append({"G": g_, "zero_point": zp, "search_ms": srch["ms"], "search_tflops": srch["value"],
                         "alpha_index": srch["best_index"], "quantize_gbs": qnt["value"], "quantize_us": qnt["us"],
                         "gemv_m1_us": round(us1, 3), "gemv_m1_gbs": round(nb1 / (us1 * 1e-6) / 1e9, 1),
                         "gemm_m512_us": round(us2, 2), "gemm_m512_tflops": round(flop2 / (us2 * 1e-6) / 1e12, 1)})
            del copies, xs, q, sc, z, Xp
            torch.cuda.empty_cache()
    awq.device_error()
    return {"workload": "quantization-sweep-4096x4096-t512-a20", "per_config": rows}


def inputs_group_sizes():
    return (32, 64, 128, 256)


def _cpu_info():
    model = platform.processor() or "unknown"
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def cpu_baseline_sample(seconds: float = 6.0):
    """The oracle, as it stands, on a bounded sample of the decode workload: the first
    256 output channels of each of the four fused linears (fp64 dequantise + matmul),
    timed with all host cores and with one thread."""
    from oracle import awq_oracle as O
    sample = []
    for name, W, X in inputs.fused_layer_inputs(1, 0.02):
        Ws = W[:256]
        q, sc, z = O.quantize_pack(Ws, None, G, ZP)
        sample.append((X, q, sc, z, W.shape[1]))
    nbytes = sum(linear_bytes(1, 256, k) for *_, k in sample)

    def run():
        t0 = time.perf_counter()
        passes = 0
        while True:
            for X, q, sc, z, K in sample:
                O.linear(X, q, sc, z, K, G, ZP)
            passes += 1
            if time.perf_counter() - t0 > seconds:
                break
        return nbytes * passes / (time.perf_counter() - t0) / 1e9, passes

    nproc, model = _cpu_info()
    all_gbs, all_passes = run()
    one_gbs, one_passes = None, 0
    threads = nproc
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
        with threadpool_limits(1):
            one_gbs, one_passes = run()
    except Exception:
        pass
    return {"value": round(all_gbs, 4), "unit": "GB/s", "cores": threads, "nproc": nproc, "cpu_model": model,
            "kind": "oracle", "single_thread_value": None if one_gbs is None else round(one_gbs, 4),
            "sample": f"first 256 output channels of each of the 4 fused linears ({nbytes} algorithmic bytes per "
                      f"pass): {all_passes} passes on {threads} threads and {one_passes} on one thread, "
                      f"{seconds:.0f} s each"}


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
    # warm-up steps (untimed): the unfused layer, then the fused layer
    unfused = build_decode_layer(awq, torch, seed_offset=rank * 100, fused=False)
    step_bytes_7 = layer_bytes(inputs.MISTRAL_7B_LAYER, 1)
    t7, steps7 = time_decode(awq, torch, unfused, args.steps, world)
    ms7 = _max_over_ranks(world, med(t7))
    launches7 = per_launch_gemv(awq, torch, unfused)
    for L in unfused:
        L.clear()
    del unfused
    torch.cuda.empty_cache()

    # headline: the layer with q/k/v and gate/up fused (4 dependent launches per step)
    layers = build_decode_layer(awq, torch, seed_offset=rank * 100, fused=True)
    step_bytes = sum(linear_bytes(1, n, k) for _, k, n, _ in inputs.MISTRAL_7B_LAYER_FUSED)
    for _ in range(args.warmup):
        for L in layers:
            awq.linear_gemv(L["x"], *L["copies"][0], G, ZP, out=L["y"])
    with ClockSampler(local) as clocks:
        trials, steps = time_decode(awq, torch, layers, args.steps, world)
    ms = _max_over_ranks(world, med(trials))
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
                "frac_spec": round(achieved / SPEC_HBM_GBS, 4),
                "per_linear_us": {n: round(t * 1e3, 2) for n, _, t in launches},
                "kernel": "gemv_tma_kernel<128, true>",
                "algorithmic_bytes_per_layer": kern_bytes}
    unfused_obj = {"workload": "mistral7b-layer-decode-gemv-m1-g128-zp-unfused",
                   "value": round(aggregate_gbs(world, step_bytes_7, steps7, ms7), 1), "unit": "GB/s",
                   "ms_per_step": round(ms7 / steps7, 5), "launches_per_step": 7,
                   "per_linear_us": {n: round(t * 1e3, 2) for n, _, t in launches7}}

    e2e_steps = max(50, min(args.steps, 400))
    eager_ms, graph_ms, h2d, d2h = time_decode_e2e(awq, torch, layers, e2e_steps)
    eager_ms = _max_over_ranks(world, eager_ms)
    graph_ms = _max_over_ranks(world, graph_ms)
    pipe_ms, pipe_graph_ms = time_decode_e2e_pipelined(awq, torch, layers, e2e_steps)
    pipe_ms = _max_over_ranks(world, pipe_ms)
    pipe_graph_ms = _max_over_ranks(world, pipe_graph_ms)
    e2e = {"value": round(aggregate_gbs(world, step_bytes, e2e_steps, pipe_graph_ms), 1), "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "how": "per step: one pinned H2D copy of the 4 input vectors, 4 awq_linear_gemv calls through the C ABI, "
                  "one D2H copy of the 4 outputs into pinned memory; the uploads and downloads run on their own "
                  "streams, overlapped with the GEMVs of the neighbouring steps (2 buffers in flight); the calls "
                  "of 8 steps captured in one CUDA graph, replayed; median of 5 trials",
           "pipelined_eager_value": round(aggregate_gbs(world, step_bytes, e2e_steps, pipe_ms), 1),
           "pipelined_eager_how": "the same pipelined steps, every call issued from Python",
           "serial_value": round(aggregate_gbs(world, step_bytes, e2e_steps, eager_ms), 1),
           "serial_how": "copies and calls in order on one stream, every call issued from Python",
           "serial_graph_value": round(aggregate_gbs(world, step_bytes, e2e_steps, graph_ms), 1),
           "serial_graph_how": "the serial step captured once per weight rotation in a CUDA graph, "
                               "one graph replay per step"}

    for L in layers:
        L.clear()
    torch.cuda.empty_cache()
    extra = {}
    if not args.skip_extra:
        extra["single_gemv"] = measure_single_gemv(awq, torch, peaks)
        extra["batched"] = measure_batched(awq, torch, peaks)
        extra["gemm"] = measure_gemm(awq, torch, peaks)
        # DRAM bytes of one launch of the o_proj-shaped linear (the captured case)
        extra["gemm"]["traffic_o_proj"] = profile_traffic("gemm_llama70b_o_proj")
        extra["quantize"] = measure_quantize(awq, torch, peaks)
        extra["quantize"]["traffic"] = profile_traffic("quantize_pack_4096")
        extra["scale_search"], _ = measure_search(awq, torch, peaks)
        extra["scale_search"]["traffic"] = profile_traffic("search_fused_4096")
        extra["scale_search_duo"], _ = measure_search(awq, torch, peaks, duo=True)
        extra["apply_clip"] = measure_clip(awq, torch, peaks)
        extra["apply_clip"]["traffic"] = profile_traffic("apply_clip_4096")
        extra["sweep"] = measure_sweep(awq, torch, peaks)

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
                           "timing": f"median of {TRIALS} trials, each {steps} steps as CUDA graph replays, "
                                     "CUDA events on the replay stream, max over ranks",
                           "trials_ms_per_step": [round(t / steps, 5) for t in trials]},
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
    nproc, model = _cpu_info()
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = nproc
    value = nbytes * args.steps / dt / 1e9
    sample_desc = f"first {rows} output channels of each of the 4 fused Mistral-7B linears per step"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "sample": sample_desc},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "nproc": nproc,
                             "cpu_model": model, "kind": "oracle", "sample": sample_desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile(args):
    """Profiling mode (no timing, no JSON): run each selected kernel a few times on its
    workload and exit; ncu selects launches from this with -k / -s / -c.
      gemv      two passes of the fused decode layer (four GEMV launches each)
      gemm      one launch of each of the four Llama-70B prefill GEMMs
      gemm_small one 2048 x 8192 x 8192 GEMM (a capture-sized case)
      gemm_m16  two 16 x 4096 x 4096 GEMMs (batched-decode size)
      quantize  three quantise/pack launches on the 4096x4096 layer
      search    two scale searches on the 4096x4096 layer with 512 tokens (G=128, zp)
      clip      two apply_clip calls on that layer (G=128, zp, 10 ratios)"""
    import torch
    from bit_weight_only_linear_b200 import awq, build
    build.build()
    awq.load_library()
    torch.cuda.set_device(0)
    what = set(args.profile.split(","))
    if "gemv" in what or "all" in what:
        layers = build_decode_layer(awq, torch, 0, fused=True)
        for _ in range(2):
            for L in layers:
                awq.linear_gemv(L["x"], *L["copies"][0], G, ZP, out=L["y"])
        torch.cuda.synchronize()
        for L in layers:
            L.clear()
        torch.cuda.empty_cache()
    if "gemm" in what or "all" in what:
        for i, (name, K, N) in enumerate(inputs.LLAMA_70B_FUSED):
            W = torch.from_numpy(inputs.weights(N, K, 0.015, inputs.SEED_W + 30 + i)).cuda()
            q, sc, z = awq.quantize_pack(W, None, G, ZP)
            del W
            X = torch.from_numpy(inputs.activations(2048, K, inputs.SEED_X + 30 + i, inputs.SEED_OUTLIER + 30)).cuda()
            awq.linear_gemm(X, q, sc, z, G, ZP)
            torch.cuda.synchronize()
            del q, sc, z, X
    if "gemm_m16" in what:
        W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W + 33)).cuda()
        q, sc, z = awq.quantize_pack(W, None, G, ZP)
        X = torch.from_numpy(inputs.activations(16, 4096, inputs.SEED_X + 33)).cuda()
        for _ in range(2):
            awq.linear_gemm(X, q, sc, z, G, ZP)
        torch.cuda.synchronize()
    if "gemm_small" in what:
        W = torch.from_numpy(inputs.weights(8192, 8192, 0.015, inputs.SEED_W + 31)).cuda()
        q, sc, z = awq.quantize_pack(W, None, G, ZP)
        X = torch.from_numpy(inputs.activations(2048, 8192, inputs.SEED_X + 31, inputs.SEED_OUTLIER + 30)).cuda()
        for _ in range(2):
            awq.linear_gemm(X, q, sc, z, G, ZP)
        torch.cuda.synchronize()
    if "quantize" in what or "all" in what:
        W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W)).cuda()
        for _ in range(3):
            awq.quantize_pack(W, None, G, ZP)
        torch.cuda.synchronize()
    if "search" in what or "all" in what:
        W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W + SWEEP_SEED_OFFSET)).cuda()
        X = torch.from_numpy(inputs.activations(512, 4096, inputs.SEED_X + SWEEP_SEED_OFFSET,
                                                inputs.SEED_OUTLIER + SWEEP_SEED_OFFSET)).cuda()
        for _ in range(2):
            awq.scale_search(X, W, G, ZP, 20)
        torch.cuda.synchronize()
    if "clip" in what or "all" in what:
        W = torch.from_numpy(inputs.weights(4096, 4096, 0.02, inputs.SEED_W + SWEEP_SEED_OFFSET)).cuda()
        X = torch.from_numpy(inputs.activations(512, 4096, inputs.SEED_X + SWEEP_SEED_OFFSET,
                                                inputs.SEED_OUTLIER + SWEEP_SEED_OFFSET)).cuda()
        s, _, _ = awq.scale_search(X, W, G, ZP, 20)
        for _ in range(2):
            awq.apply_clip(X, W, s, G, ZP, 20, 10)
        torch.cuda.synchronize()
    awq.device_error()
    print("profile run done", flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--skip-extra", action="store_true", help="headline decode measurement only")
    ap.add_argument("--skip-cpu", action="store_true", help="do not time the CPU oracle")
    ap.add_argument("--profile", default=None,
                    help="no timing: run the named kernels (gemv,gemm,gemm_small,quantize,search,all) for ncu")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile:
        run_profile(args)
        return
    if args.impl == "reference":
        if args.steps == 200:
            args.steps = 20
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
