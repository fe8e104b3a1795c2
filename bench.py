#!/usr/bin/env python
"""Throughput of the sparse MoE feed-forward layer on B200 (one JSON line).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole layer (router, permutation, routed experts,
shared expert, combine) over one batch of synthetic tokens already resident in
HBM.  Default workload: the Talker decode layer (T=8 tokens, hidden 1024, 128
experts Top-6, experts 1024->384->1024, shared 1024->768->1024, bf16).  To keep
weights from being served out of the 126 MB L2, decode steps cycle through 8
independent weight copies (2.46 GB); prefill steps touch >300 MB each anyway.

The timed loop replays CUDA graphs of captured forward calls (the same kernels a
forward launches; graphs remove per-call host overhead), exactly --steps of them.  With N > 1 (torchrun)
every rank runs its own replica on its own tokens (weak scaling, no collective
on the data path); the time is the max over ranks.

Reported besides the device throughput:
  e2e           the same metric through moe_forward_host (host buffers, the
                host->device and device->host copies inside the timed region)
  roofline      routed-expert kernel: algorithmic bytes (touched expert weights +
                its input and output rows) or FLOPs per launch / its mean
                CUDA-event duration, against MEASURED_PEAKS.json
  cpu_baseline  the fp64 oracle on this host's cores over a bounded sample (and on
                one thread over half that time), with the CPU model
  clocks        nvidia-smi samples taken during the timed loop
  env           GPU name, driver, CUDA runtime, torch and library versions
--impl reference times the oracle alone (the CPU reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from concurrent.futures import ThreadPoolExecutor
from datetime import timedelta

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s on 1 B200; % of HBM (decode) / tensor (prefill) roofline"
ROTATE = {"talker_decode": 8, "tiny_fp32": 1, "talker_prefill": 1,
          "talker_prefill_skewed": 1, "talker_stack20": 1}
DEFAULT_STEPS = {"talker_decode": 20000, "tiny_fp32": 20000, "talker_prefill": 400,
                 "talker_prefill_skewed": 100, "talker_stack20": 200}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


# ----------------------------------------------------------------------------- setup
def parse():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="talker_decode", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--rotate", type=int, default=None, help="independent weight copies")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="CPU work of the oracle baseline sample")
    ap.add_argument("--no-graph", action="store_true", help="time eager calls, not graphs")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    return ap.parse_args()


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def load_peaks(path=None):
    """Measured HBM copy bandwidth and bf16 GEMM throughput of this GPU model, else the
    fallback figures (an unreadable or incomplete file counts as absent)."""
    p = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        hbm, tf = float(d["hbm_gbs"]), float(d["bf16_tflops"])
        if hbm > 0 and tf > 0:
            return {"hbm_gbs": hbm, "bf16_tflops": tf,
                    "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                    "source": "measured"}
    except (OSError, ValueError, KeyError, TypeError):
        pass
    return dict(FALLBACK_PEAKS)


def source_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(workload, kernel):
    """DRAM bytes per launch of the roofline kernel from a committed ncu summary,
    valid only while that kernel's source file is unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel") != kernel:
        return None
    src = os.path.join(ROOT, "sparse_moe_transformer_b200", "csrc", e["source"])
    if not os.path.exists(src) or e.get("source_sha") != source_sha(src):
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of the GPU's clocks and throttle reasons (every 100 ms)."""
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != 6:
                continue
            try:
                sm.append(float(parts[0])); mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[2:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def run_env(torch, dev, smt, gpu_uuid):
    """Run conditions: GPU name, driver, CUDA runtime, torch and library versions
    (None for anything that cannot be read)."""
    def driver():
        r = subprocess.run(["nvidia-smi", "-i", gpu_uuid, "--query-gpu=driver_version",
                            "--format=csv,noheader"], capture_output=True, text=True, timeout=20)
        return r.stdout.strip() or None
    env = {}
    for key, fn in (("gpu", lambda: torch.cuda.get_device_name(dev)), ("driver", driver),
                    ("cuda_runtime", lambda: torch.version.cuda),
                    ("torch", lambda: torch.__version__), ("library", lambda: smt.version())):
        try:
            env[key] = fn()
        except Exception:
            env[key] = None
    return env


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Largest value across ranks (the timing rule: the slowest rank sets the time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- workloads
def build_inputs(name, rank, rotate):
    """Per-copy (layers, x, residual) lists; copy 0 of rank 0 is the canonical input."""
    wl = synth.WORKLOADS[name]
    base = synth.make(name)
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        extra = list(ex.map(lambda r: synth.make_extra_weights(name, r), range(1, rotate)))
    copies = []
    for r in range(rotate):
        layers = base.layers if r == 0 else [extra[r - 1]]
        x = base.x if (r == 0 and rank == 0) else synth.make_tokens(wl, base.x.shape[0],
                                                                    seed=rank * 1000 + r)
        copies.append((layers, x))
    return wl, copies


def algorithmic_work(wl, idx_list, residual=False):
    """Per-step algorithmic bytes / FLOPs of the whole layer and of the routed-expert
    kernel, from the realised routing (weights of experts with >= 1 token); a residual
    input adds its T x H read."""
    H, E, k, I, Is = wl.H, wl.E, wl.k, wl.I, wl.Is
    es = 2 if wl.dtype == "bf16" else 4
    out = []
    for idx in idx_list:
        T = idx.shape[0]
        touched = int(np.unique(idx).size)
        experts_bytes = touched * 3 * H * I * es + 2 * T * k * H * es
        act_rows = 3 if residual else 2          # x, y (and the residual)
        layer_bytes = (es * (H * E + touched * 3 * H * I + 3 * H * Is + act_rows * T * H)
                       + T * k * 8)
        experts_flops = 2 * 3 * H * I * T * k
        layer_flops = T * (2 * H * E + k * 2 * 3 * H * I + 2 * 3 * H * Is)
        out.append(dict(touched=touched, experts_bytes=experts_bytes, layer_bytes=layer_bytes,
                        experts_flops=experts_flops, layer_flops=layer_flops))
    return out


def graph_plan(K, rotate, per_graph=32):
    """How CUDA graphs time exactly K steps: a graph of `cycle` steps (whole rotation
    cycles of the weight copies when K allows; step i uses copy i % rotate) replayed
    n_rep times, then a graph of the remaining `rem` steps (starting again at copy 0)."""
    if K < 1:
        raise ValueError("--steps must be >= 1")
    cycle = min(K, rotate * max(1, per_graph // rotate))
    n_rep, rem = divmod(K, cycle)
    return cycle, n_rep, rem


# ----------------------------------------------------------------------------- CPU arms
def cpu_model():
    """The host CPU's model name (Linux), or None."""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def oracle_sample_rate(wl, layers, x, seconds, nthreads=None):
    """Tokens/s of the fp64 oracle on this host's cores (or on `nthreads` threads) over
    a bounded sample (whole token batches until `seconds` have passed)."""
    import oracle
    cores = nthreads or len(os.sched_getaffinity(0))
    T = x.shape[0]
    n_tok = T if wl.n_layers > 1 or T <= 64 else 64
    xs = x[:n_tok]
    orcs = [oracle.Oracle(oracle.LayerWeights(**L.arrays(), top_k=wl.k, rms_eps=wl.rms_eps))
            for L in layers]
    done, t0 = 0, time.perf_counter()
    while True:
        h = xs
        for o in orcs:
            y, _, _, _ = o.forward(h, residual=h if wl.n_layers > 1 else None, nthreads=cores)
            h = synth.bf16_bits(y) if wl.dtype == "bf16" else y.astype(np.float32)
        done += n_tok
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    threads = orcs[0].threads(cores)
    sample = (f"{done} tokens ({n_tok}-token batches of the {wl.name} inputs, "
              f"{len(orcs)} layer(s)) in {dt:.1f} s")
    return done / dt, threads, sample


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    name = args.workload
    wl = synth.WORKLOADS[name]
    base = synth.make(name)
    K = args.steps if args.steps is not None else 5
    W = args.warmup if args.warmup is not None else 1
    import oracle
    cores = len(os.sched_getaffinity(0))
    T = base.x.shape[0]
    n_tok = T if wl.n_layers > 1 or T <= 64 else 64
    orcs = [oracle.Oracle(oracle.LayerWeights(**L.arrays(), top_k=wl.k, rms_eps=wl.rms_eps))
            for L in base.layers]

    def step():
        h = base.x[:n_tok]
        for o in orcs:
            y, _, _, _ = o.forward(h, residual=h if wl.n_layers > 1 else None, nthreads=cores)
            h = synth.bf16_bits(y) if wl.dtype == "bf16" else y.astype(np.float32)

    for _ in range(W):
        step()
    t0 = time.perf_counter()
    for _ in range(K):
        step()
    dt = time.perf_counter() - t0
    value = n_tok * K / dt
    threads = orcs[0].threads(cores)
    sample = f"{n_tok} of the {T} tokens of {name} per step, {K} steps"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": dt / K * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(wl, world, 1, "fp64 oracle on host cores"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(wl, world, rotate, l2):
    return {"workload": wl.name, "tokens_per_gpu": wl.T, "global_batch": wl.T * world,
            "hidden": wl.H, "experts": wl.E, "top_k": wl.k, "expert_inter": wl.I,
            "shared_inter": wl.Is, "layers": wl.n_layers, "pre_rmsnorm": wl.rms,
            "parallelism": f"replicas x{world}", "weight_copies": rotate, "l2": l2}


# ----------------------------------------------------------------------------- GPU arm
def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist
    import sparse_moe_transformer_b200 as smt
    from sparse_moe_transformer_b200 import build as smt_build
    smt_build.build()           # no-op when the in-tree library is up to date

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device(f"cuda:{local}"))
    name = args.workload
    rotate = args.rotate or ROTATE[name]
    K = args.steps if args.steps is not None else DEFAULT_STEPS[name]
    W = args.warmup if args.warmup is not None else max(3, min(200, K // 10))
    wl, copies = build_inputs(name, rank, rotate)
    cfg = smt.LayerConfig(wl.H, wl.E, wl.k, wl.I, wl.Is, wl.dtype, wl.rms_eps)
    T = wl.T
    dev = torch.device(f"cuda:{local}")
    stream = torch.cuda.Stream(device=dev)

    # upload: one handle per (copy, layer); inputs and outputs resident in HBM
    handles, xs, ys = [], [], []
    for layers, x in copies:
        hs = [smt.MoELayer.from_numpy(cfg, L.arrays(), device=local, max_tokens=T)
              for L in layers]
        handles.append(hs)
        xs.append(smt.to_device(x, local))
        ys.append([torch.empty_like(xs[-1]) for _ in hs])
    stack = wl.n_layers > 1

    def step(r):
        h = xs[r]
        for li, layer in enumerate(handles[r]):
            layer.forward(h, residual=h if stack else None, out=ys[r][li], stream=stream)
            h = ys[r][li]

    # realised routing of each copy (for algorithmic bytes)
    idx_list = []
    with torch.cuda.stream(stream):
        for r in range(rotate):
            h = xs[r]
            for li, layer in enumerate(handles[r]):
                y, idx, _ = layer.forward(h, residual=h if stack else None, return_routing=True,
                                          stream=stream)
                idx_list.append(idx.cpu().numpy())
                h = y
    torch.cuda.synchronize()
    work = algorithmic_work(wl, idx_list, residual=stack)
    for hs in handles:
        for layer in hs:
            st = layer.check(stream)
            assert st == 0, f"device-side status {st}"

    # ---- warm-up, then CUDA graphs that together hold exactly K steps
    for i in range(W):
        with torch.cuda.stream(stream):
            step(i % rotate)
    torch.cuda.synchronize()
    use_graph = not args.no_graph
    cycle, n_rep, rem = graph_plan(K, rotate)
    graph = graph_rem = None
    launches_per_step = 0.0
    if use_graph:
        for hs in handles:
            for layer in hs:
                layer.kernel_stats(reset=True)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for i in range(cycle):
                step(i % rotate)
        # every launch the library made while capturing is a kernel node of the graph
        launches_per_step = sum(n for hs in handles for layer in hs
                                for n, _ in layer.kernel_stats(reset=True).values()) / cycle
        if rem:
            graph_rem = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_rem, stream=stream):
                for i in range(rem):
                    step(i % rotate)
        with torch.cuda.stream(stream):
            graph.replay()
            if graph_rem is not None:
                graph_rem.replay()
        torch.cuda.synchronize()
    steps_timed = K
    for hs in handles:
        for layer in hs:
            layer.kernel_stats(reset=True)

    gpu_uuid = str(torch.cuda.get_device_properties(dev).uuid)
    gpu_uuid = gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}"
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(gpu_uuid) as clocks:
        start.record(stream)
        if use_graph:
            with torch.cuda.stream(stream):      # replay on the stream the events time
                for _ in range(n_rep):
                    graph.replay()
                if graph_rem is not None:
                    graph_rem.replay()
        else:
            with torch.cuda.stream(stream):
                for i in range(K):
                    step(i % rotate)
        end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(end)
    t_max = max_over_ranks(ms, dist, dev)
    launches = int(round(launches_per_step * steps_timed))
    value = world * T * steps_timed / (t_max / 1e3)
    for hs in handles:
        for layer in hs:
            layer.kernel_stats(reset=True)

    # ---- per-kernel durations (events around each launch on its own stream); bursts
    # queued behind a spin kernel so host enqueue time does not enter the kernels' spans
    kt_steps = min(steps_timed, 400)
    for hs in handles:
        for layer in hs:
            layer.set_option("kernel_timing", 1)
    done = 0
    while done < kt_steps:
        burst = min(8, kt_steps - done)
        with torch.cuda.stream(stream):
            torch.cuda._sleep(20_000_000)        # ~10 ms: covers the burst's host enqueue
            for i in range(burst):
                step((done + i) % rotate)
        done += burst
    torch.cuda.synchronize()
    per_class = {}
    for hs in handles:
        for layer in hs:
            for c, (n, t) in layer.kernel_stats(reset=True).items():
                a = per_class.setdefault(c, [0, 0.0])
                a[0] += n
                a[1] += t
            layer.set_option("kernel_timing", 0)
    if not use_graph:
        launches = sum(v[0] for v in per_class.values()) * K // max(1, kt_steps)
    kern = {c: {"launches": n, "mean_us": (t / n * 1e3) if n else None}
            for c, (n, t) in per_class.items()}

    # ---- per-call latency: one single-call graph per weight copy, each replay between
    # two events on the bench stream (device time of one forward call; p50/p95/p99)
    lat = None
    if use_graph:
        one = []
        for r in range(rotate):
            g1 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g1, stream=stream):
                step(r)
            one.append(g1)
        n_lat = min(400, max(20, steps_timed))
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_lat)]
        with torch.cuda.stream(stream):
            for i, (e0, e1) in enumerate(evs):
                e0.record(stream)
                one[i % rotate].replay()
                e1.record(stream)
        torch.cuda.synchronize()
        us = np.array([e0.elapsed_time(e1) * 1e3 for e0, e1 in evs])
        lat = {"p50": float(np.percentile(us, 50)), "p95": float(np.percentile(us, 95)),
               "p99": float(np.percentile(us, 99)), "unit": "us", "calls": n_lat,
               "what": "device time of one call, single-call CUDA graph between events"}
        del one
    for hs in handles:
        for layer in hs:
            layer.kernel_stats(reset=True)

    # ---- roofline of the dominant kernel (the expert kernel)
    peaks = load_peaks()
    ex_n, ex_ms = per_class.get("experts", (0, 0.0))
    ex_s = (ex_ms / ex_n) / 1e3 if ex_n else None
    e_bytes = float(np.mean([w["experts_bytes"] for w in work]))
    e_flops = float(np.mean([w["experts_flops"] for w in work]))
    # no shared-expert launch: the expert kernel's tiles include the shared expert
    # (its weights once, every token); no permutation either: the few-token kernel
    few_token = per_class.get("permute", (0, 0))[0] == 0
    if wl.Is and per_class.get("shared", (0, 0))[0] == 0:
        es = 2 if wl.dtype == "bf16" else 4
        e_bytes += 3 * wl.H * wl.Is * es + (0 if few_token else 2 * T * wl.H * es)
        e_flops += 2 * 3 * wl.H * wl.Is * T
    kname = "tc_fused_experts_kernel" if few_token else "tc_routed_experts_kernel"
    t_mem = e_bytes / (peaks["hbm_gbs"] * 1e9)
    t_tc = e_flops / (peaks["bf16_tflops"] * 1e12)
    if ex_s:
        if t_mem >= t_tc:
            achieved = e_bytes / ex_s / 1e9
            roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"]}
        else:
            achieved = e_flops / ex_s / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"]}
        roof["traffic"] = recorded_traffic(name, kname)
        roof["kernel"] = kname + (" (few-token tiles: routed + shared experts, h on chip)"
                                  if few_token else " (grouped routed + shared expert tiles)")
        roof["algorithmic_per_launch"] = e_bytes if roof["bound"] == "hbm" else e_flops
        roof["mean_launch_us"] = ex_s * 1e6
        roof["peak_source"] = peaks["source"] + (" burst" if roof["bound"] == "tensor" else "")
    else:
        roof = None
    layer_bytes = float(np.mean([w["layer_bytes"] for w in work])) * wl.n_layers
    layer_flops = float(np.mean([w["layer_flops"] for w in work])) * wl.n_layers
    step_s = t_max / 1e3 / steps_timed
    whole = {"alg_bytes_per_step": layer_bytes, "alg_flops_per_step": layer_flops,
             "achieved_GBps": layer_bytes / step_s / 1e9,
             "achieved_TFLOPs": layer_flops / step_s / 1e12,
             "roofline_frac": max(layer_bytes / (peaks["hbm_gbs"] * 1e9),
                                  layer_flops / (peaks["bf16_tflops"] * 1e12)) / step_s,
             "touched_experts_mean": float(np.mean([w["touched"] for w in work]))}

    # ---- end to end through the public host-buffer API
    K_e2e = min(steps_timed, 2000 if T <= 64 else 50)
    es = 2 if wl.dtype == "bf16" else 4
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    xh = [smt.to_numpy(x) for x in xs]
    xh = [torch.from_numpy(a.view(np.int16) if a.dtype == np.uint16 else a).view(tdt).pin_memory()
          for a in xh]
    yh = torch.empty_like(xh[0]).pin_memory()
    h2d = d2h = T * wl.H * es
    for i in range(3):
        e2e_step(handles[i % rotate], xh[i % rotate], yh, stream, stack, dev)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s2.record(stream)
    for i in range(K_e2e):
        e2e_step(handles[i % rotate], xh[i % rotate], yh, stream, stack, dev)
    e2.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(s2.elapsed_time(e2), dist, dev)
    e2e = {"value": world * T * K_e2e / (e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "steps": K_e2e, "api": "moe_forward_host (pinned host buffers)"}

    # ---- CPU baseline (oracle), rank 0 at N=1 only
    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        v, threads, sample = oracle_sample_rate(wl, copies[0][0], copies[0][1], args.cpu_seconds)
        v1, _, sample1 = oracle_sample_rate(wl, copies[0][0], copies[0][1],
                                            args.cpu_seconds / 2, nthreads=1)
        cpu = {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": sample, "cpu_model": cpu_model(),
               "single_thread": {"value": v1, "unit": "tokens/s", "sample": sample1}}

    for hs in handles:
        for layer in hs:
            assert layer.check(stream) == 0
    del graph, graph_rem
    if rank == 0:
        l2 = (f"rotate {rotate} independent weight copies ({rotate * copies[0][0][0].nbytes / 1e9:.2f}"
              f" GB) > 126 MB L2" if rotate > 1 else
              f"inputs larger than L2 ({whole['alg_bytes_per_step'] / 1e6:.0f} MB touched per step)")
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": steps_timed, "warmup": W, "ms_per_step": t_max / steps_timed,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": wl.dtype, "data": "synthetic (seeded; random-init weights)",
                "impl": "ours", "config": workload_config(wl, world, rotate, l2),
                "timing": "CUDA graphs of captured forward calls" if use_graph else "eager",
                "roofline": roof, "layer": whole, "kernels": kern, "latency": lat,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
                "clocks": clocks.summary(), "env": run_env(torch, dev, smt, gpu_uuid)}
        print(json.dumps(line), flush=True)
    for hs in handles:
        for layer in hs:
            layer.close()
    if world > 1:
        dist.destroy_process_group()


def e2e_step(layers, xh, yh, stream, stack, dev):
    if not stack:
        layers[0].forward_host(xh, yh, stream=stream)
        return
    # a stack step: host input in, 20 device-resident layers, host output back
    import torch
    with torch.cuda.stream(stream):
        h = xh.to(dev, non_blocking=True)
        for layer in layers:
            h = layer.forward(h, residual=h, stream=stream)
        yh.copy_(h, non_blocking=True)
    stream.synchronize()


if __name__ == "__main__":
    main()
