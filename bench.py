#!/usr/bin/env python
"""Benchmark of the routed-MoE FFN path on B200.

Default workload (the headline): the 48-layer decode stack (512 Q2 experts
per layer, hidden 2048, intermediate 768, top-10, one token per step, residual
RMSNorm), one CUDA graph replay per token, timed with CUDA events over K
steps after W warm-up steps. The same JSON line then carries two more seeds of
that workload and the other workloads, each measured on freshly generated
weights with its own roofline, clocks and CPU-oracle baseline:

  config1_layer    one Q2 decode layer, one token; steps cycle over 16 layers (weights > L2)
  config3_verify   8 correlated tokens through 48 Q4 layers (verify batch)
  config4_prefill  a 4096-token bf16 chunk through one Q4 layer
  mixed48_decode   the 48-layer single-token stack with every fourth layer in Q4
                   (mixed-bit stack: the fused kernel takes each layer's format)
  ngram_gather     16 hashed rows per token of a 2^22 x 256 Q4 n-gram table, 4096 tokens

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode48|verify48|mixed48|layer|prefill|ngram] [--headline-only]

N > 1 runs N independent replicas (one process per GPU under torchrun; the
path has no exchange step), timed on the device, max over ranks.
"""
from __future__ import annotations

import argparse
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

METRIC = "MoE decode tokens/s over 48 layers; HBM GB/s on weight bytes vs peak"
PREFILL_METRIC = "MoE prefill tokens/s (4096-token bf16 chunk, one 512-expert Q4 layer); tensor TFLOP/s vs peak"
SEED = 0
LAYER_CYCLE = 16      # distinct layers the single-layer steps cycle over (weights > L2)
WORKLOADS = {"decode48": 2, "verify48": 3, "mixed48": 2, "layer": 1, "prefill": 4, "ngram": None}
NGRAM_METRIC = ("n-gram row gather tokens/s (16 hashed rows of a 2^22 x 256 Q4 table per token, 4096-token "
                "chunk); HBM GB/s on row and output bytes vs peak")
MIXED_EVERY = 4       # mixed48: layers 0, 4, 8, ... in Q4, the others in Q2


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="decode48", choices=sorted(WORKLOADS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--headline-only", action="store_true",
                   help="decode48: only the 48-layer single-token stack (no extra seeds, no other workloads)")
    p.add_argument("--layers", type=int, default=None,
                   help="decode workloads only: layers in the stack (default: all 48); for small profiling runs")
    p.add_argument("--tokens", type=int, default=None,
                   help="prefill workload only: tokens per chunk (default: the workload's 4096)")
    return p.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s for a kernel timed per launch (about half a
    millisecond, not inside a seconds-long loop): the burst figure."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured (burst)"
    return 1590.0, "fallback (burst)"


def format_desc(cfg):
    if not cfg.fmt_layers:
        return f"Q{cfg.fmt}"
    n4 = sum(1 for f in cfg.fmt_layers if f == 4)
    return f"mixed: Q4 in {n4} of {cfg.L} layers (every {MIXED_EVERY}th from layer 0), Q2 in the rest"


def workload_desc(cfg, T):
    return {"workload": f"{cfg.L}-layer routed-MoE decode stack: {cfg.E} experts/layer, hidden {cfg.H}, "
                        f"intermediate {cfg.I}, top-{cfg.k}, {format_desc(cfg)} blocks, {T} token(s)/step, "
                        f"residual RMSNorm",
            "layers": cfg.L, "experts_per_layer": cfg.E, "hidden": cfg.H, "intermediate": cfg.I, "top_k": cfg.k,
            "format": format_desc(cfg), "tokens_per_step": T, "seed": SEED,
            "l2": "no flush: each step streams ~0.85-3.5 GB of distinct experts (> 126 MB L2); "
                  "a fresh token is drawn for every step"}


# ------------------------------------------------------------------ clocks --
REASON_BITS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))


def summarize_clock_samples(samples, max_mhz):
    """samples: (sm_mhz, reason_bitmask) pairs taken during a timed region."""
    if not samples:
        return {"sm_mhz": None, "sm_max_mhz": max_mhz, "reasons": ["no samples"], "samples": 0}
    reasons = sorted({n for _, r in samples for n, bit in REASON_BITS if r & bit})
    return {"sm_mhz": statistics.median(m for m, _ in samples), "sm_max_mhz": max_mhz, "reasons": reasons,
            "samples": len(samples), "sm_mhz_min": min(m for m, _ in samples)}


class NvmlClocks:
    """SM clock and throttle reasons sampled through NVML every ~2 ms on a
    host thread while the timed region runs (several samples even for a
    region of a few tens of milliseconds)."""

    def __init__(self, dev_uuid, period_s=0.002):
        import threading

        import pynvml
        pynvml.nvmlInit()
        self.nv = pynvml
        self.h = pynvml.nvmlDeviceGetHandleByUUID(dev_uuid)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.samples = []
        self.period = period_s
        self.stop_ev = threading.Event()
        self.t = threading.Thread(target=self._run, daemon=True)
        self.t.start()

    def _run(self):
        nv = self.nv
        while not self.stop_ev.is_set():
            try:
                self.samples.append((float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)),
                                     int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))))
            except Exception:
                pass
            time.sleep(self.period)

    def stop(self):
        self.stop_ev.set()
        self.t.join(timeout=5)
        return summarize_clock_samples(self.samples, self.max_mhz)


class Clocks:
    """Fallback sampler: nvidia-smi at 100 ms."""
    Q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_uuid):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        self.f = os.fdopen(fd, "w")
        args = ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits", "-lms", "100"]
        if dev_uuid:
            args[1:1] = ["-i", dev_uuid]
        try:
            self.p = subprocess.Popen(args, stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def clock_sampler(local):
    import torch
    props = torch.cuda.get_device_properties(local)
    uuid = getattr(props, "uuid", None) and f"GPU-{props.uuid}"
    try:
        return NvmlClocks(uuid)
    except Exception:
        return Clocks(uuid)


# ---------------------------------------------------------- dist helpers --
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(v, world):
    """Maximum of a per-rank value (a device-timed duration) over all ranks."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cpu" if dist.get_backend() == "gloo" else "cuda"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world, steps, units_per_step, ms_max):
    """Whole-job throughput of N replicas: units all ranks processed / the slowest rank's time."""
    return world * steps * units_per_step / (ms_max / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ traffic file --
TRAFFIC_PROFILES = {
    # kernel -> (committed ncu summary, sources that define the kernel)
    "stack_decode": ("stack_decode_decode48_ncu.md",
                     ("stack_decode.cu", "decode_tile.cuh", "common.cuh", "layout.cuh", "route_common.cuh",
                      "decode_canon.cuh")),
    "pf_gemm1": ("pf_gemm_prefill4096_ncu.md", ("prefill.cu", "tc05.cuh", "common.cuh", "layout.cuh")),
    "ngram_gather": ("ngram_gather_ngram4096_ncu.md", ("ngram.cu", "common.cuh")),
    # per algorithmic byte (a launch's bytes depend on its routes): scaled to the measured launches
    "stack_decode_mixed": ("stack_decode_mixed48_ncu.md",
                           ("stack_decode.cu", "decode_tile.cuh", "common.cuh", "layout.cuh", "route_common.cuh",
                            "decode_canon.cuh")),
    "ffn_decode_t8": ("ffn_decode_verify8_ncu.md",
                      ("ffn_decode.cu", "decode_tile.cuh", "common.cuh", "layout.cuh", "decode_canon.cuh")),
    "ffn_decode_t1": ("ffn_decode_layer1_ncu.md",
                      ("ffn_decode.cu", "decode_tile.cuh", "common.cuh", "layout.cuh", "decode_canon.cuh")),
}


def kernel_source_hash(names):
    h = hashlib.sha256()
    for name in names:
        with open(os.path.join(ROOT, "quantised_expert_decode_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def stored_traffic(kernel, key="dram_bytes_per_launch"):
    """DRAM bytes per launch (or per algorithmic byte) from the committed ncu
    summary, if the kernel's sources have not changed since the counters were
    taken (else None)."""
    if kernel not in TRAFFIC_PROFILES:
        return None
    fname, sources = TRAFFIC_PROFILES[kernel]
    path = os.path.join(ROOT, "profiles", fname)
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if line.startswith("- ") and ":" in line:
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != kernel_source_hash(sources):
        return None
    try:
        return float(vals[key])
    except (KeyError, ValueError):
        return None


def scaled_traffic(kernel, algorithmic_bytes):
    """DRAM bytes of a launch of `algorithmic_bytes`, from a committed capture's
    traffic per algorithmic byte (the launch reads what its routes select)."""
    r = stored_traffic(kernel, "dram_bytes_per_algorithmic_byte")
    return None if r is None else r * float(algorithmic_bytes)


# --------------------------------------------------------- oracle timing --
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_token_time(cfg, x0, n_layers):
    """Seconds the float64 oracle takes for one step over n_layers (routing,
    dequantisation, expert FFNs, combine, residual RMSNorm). Weight bytes are
    drawn from the generator before each timed layer and are not counted."""
    import numpy as np
    from oracle import moe
    from synth import gen
    x = x0.astype(np.float64)
    spent = 0.0
    for l in range(n_layers):
        bits = cfg.for_layer(l).format.bits
        Wr, b = gen.router(SEED, cfg, l), gen.bias(SEED, cfg, l)
        t0 = time.perf_counter()
        idx, g, _ = moe.route(x, Wr, b, cfg.k)
        spent += time.perf_counter() - t0
        raw = {int(e): gen.expert(SEED, cfg, l, int(e)) for e in set(idx.ravel().tolist())}
        t0 = time.perf_counter()

        def get(e):
            r = raw[e]
            return tuple(moe.dequantize(r[n + "_codes"], r[n + "_scales"], bits) for n in ("gate", "up", "down"))
        y = moe.moe_layer(x, idx, g, get)
        x = moe.rmsnorm_residual(x, y, cfg.eps)
        spent += time.perf_counter() - t0
    return spent


def cpu_baseline(cfg, T, n_layers=None, repeats=1):
    """The oracle on the host cores over ``n_layers`` layers of one step
    (default: all layers for one token, 2 layers for a batch), ``repeats``
    times, scaled to the workload's layer count."""
    from synth import gen
    n = n_layers if n_layers else (cfg.L if T == 1 else 2)
    s = sum(oracle_token_time(cfg, gen.tokens(SEED, cfg, r), n) for r in range(repeats))
    tok_s = repeats * T / (s * cfg.L / n)
    return {"value": tok_s, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{repeats} step(s) of {T} token(s) through {n} of {cfg.L} layer(s) (float64 NumPy, weight "
                      f"generation excluded), scaled to {cfg.L} layer(s); {s:.1f} s of CPU work"}


# -------------------------------------------------------------- reference --
def run_reference(args, cfg, T):
    """The oracle timed as the reference arm: a step is one expert FFN of one
    token slot (1/k of a layer; the layer's routing is charged to its first
    step, its combine + RMSNorm to its last)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import numpy as np
    from oracle import moe
    from synth import gen
    x = gen.tokens(SEED, cfg, 0).astype(np.float64)
    state = {"l": 0, "idx": None, "g": None, "raw": None, "outs": {}}

    def step():
        l = state["l"] % cfg.L
        j = len(state["outs"])
        t = 0.0
        if j == 0:
            Wr, b = gen.router(SEED, cfg, l), gen.bias(SEED, cfg, l)
            t0 = time.perf_counter()
            idx, g, _ = moe.route(state.get("x", x), Wr, b, cfg.k)
            t += time.perf_counter() - t0
            state["idx"], state["g"] = idx, g
        e = int(state["idx"][0, j])
        raw = gen.expert(SEED, cfg, l, e)
        bits = cfg.for_layer(l).format.bits
        t0 = time.perf_counter()
        W = tuple(moe.dequantize(raw[n + "_codes"], raw[n + "_scales"], bits) for n in ("gate", "up", "down"))
        xx = state.get("x", x)
        state["outs"][j] = moe.expert_ffn(xx[:1], *W)[0]
        if j == cfg.k - 1:
            y = moe.combine(np.stack([state["outs"][i] for i in range(cfg.k)]), state["g"][0])
            state["x"] = moe.rmsnorm_residual(xx[:1], y[None], cfg.eps)
            state["outs"] = {}
            state["l"] += 1
        t += time.perf_counter() - t0
        return t

    for _ in range(args.warmup):
        step()
    spent = sum(step() for _ in range(args.steps))
    tokens = args.steps / (cfg.L * cfg.k)
    value = tokens / spent
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * spent / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_desc(cfg, 1),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{args.steps} steps of one expert FFN each (1/{cfg.k} of a layer of one "
                                       f"token), weight generation excluded"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- ours --
def init_dist(local, world):
    import torch
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        if not dist.is_initialized():
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))


def free_device():
    import gc
    import torch
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def measure_stack(args, cfg, seed=SEED, full=True):
    """One graph replay per step of the decode stack: device-resident inputs
    (value), the host-buffer entry point (e2e) and, with ``full``, per-kernel
    event timing for the roofline. Returns the line's fields."""
    import numpy as np
    import torch

    from quantised_expert_decode_b200.model import DecodeStack
    from synth import gen
    from synth.workload import device_layers

    rank, world, local = dist_env()
    T = cfg.T
    layers, routers, biases = device_layers(seed, cfg)
    stack = DecodeStack(layers, routers, biases, T, cfg.k, cfg.eps)
    n_in = min(args.steps + args.warmup, 4096)
    xs_host = np.stack([gen.tokens(seed + 1000 * rank, cfg, st) for st in range(n_in)])   # [n, T, H]
    xs = torch.from_numpy(xs_host).cuda()
    stream = torch.cuda.current_stream()

    def step(i):
        stack.x_in.copy_(xs[i % n_in], non_blocking=True)
        stack.decode(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    if stack.status() != 0:
        raise RuntimeError("device status set during warm-up")
    clocks = clock_sampler(local)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    value = replica_throughput(world, args.steps, T, ms)
    if stack.status() != 0:
        raise RuntimeError("device status set during the timed run")
    idx = stack.idx.cpu().numpy()
    uniq = [len(set(idx[l].ravel().tolist())) for l in range(cfg.L)]
    out = {"value": value, "ms_per_step": ms / args.steps, "clocks": clk,
           "gpu_launches": args.steps * stack.kernels_per_replay, "seed": seed}
    if not full:
        stack.close()
        del stack, layers, routers, biases, xs
        free_device()
        return out

    # end to end through the host-buffer entry point (pinned memory)
    xh = torch.from_numpy(xs_host).pin_memory()
    outh = torch.empty((T, cfg.H), dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()
    barrier(world)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for i in range(args.steps):
        stack.decode_host(xh[i % n_in], outh, stream)
    e3.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3), world)
    if stack.status() != 0:
        raise RuntimeError("device status set during the e2e run")
    stack.close()

    # kernel durations: the same steps through a graph with event nodes around
    # every route and FFN node (event nodes split the programmatic edges, so
    # this graph is timed apart from the headline); the mean over the replays
    tstack = DecodeStack(layers, routers, biases, T, cfg.k, cfg.eps, timing=True)
    for i in range(args.warmup):
        tstack.x_in.copy_(xs[i % n_in], non_blocking=True)
        tstack.decode(stream)
    torch.cuda.synchronize()
    route_ms = np.zeros(cfg.L)
    ffn_ms = np.zeros(cfg.L)
    n_t = args.steps
    for i in range(n_t):
        tstack.x_in.copy_(xs[(args.warmup + i) % n_in], non_blocking=True)
        tstack.decode(stream)
        r, f = tstack.layer_times()
        route_ms += np.asarray(r)
        ffn_ms += np.asarray(f)
    route_ms /= n_t
    ffn_ms /= n_t
    if tstack.status() != 0:
        raise RuntimeError("device status set during the timing-graph run")
    fused = tstack.path == 1
    phases = None
    if fused:
        # median CTA's clock at each phase point of a layer, from the layer's
        # start, averaged over the layers of the last replay (in microseconds
        # at the sampled SM clock)
        tr = tstack.phase_trace().astype(np.float64)                     # [L, CTAs, points]
        rows = np.arange(tr.shape[1]) < cfg.H // 16                     # CTAs with a phase D
        busy = tr[:, :, 8] != 0                                          # CTAs with gate/up tiles
        first = np.array([[np.median((tr[l, :, 8] - tr[l, :, 0])[busy[l]])] for l in range(tr.shape[0])])
        rel = np.concatenate([np.median(tr[:, :, 1:8] - tr[:, :, :1], axis=1), first,
                              np.median(tr[:, rows, 9:] - tr[:, rows, :1], axis=1)], axis=1).mean(axis=0)
        mhz = clk.get("sm_mhz") or clk.get("sm_max_mhz") or 1965.0
        names = ["topk_done", "tiles_start", "tiles_done", "barrier1_passed", "down_done", "barrier2_passed",
                 "logits_ready", "first_tile_landed", "h_limbs_landed", "down_tiles_done", "z_written"]
        phases = {n: float(v) / mhz for n, v in zip(names, rel)}
        # the slowest CTA's gate/up tiles hold the first grid barrier
        phases["tiles_done_max_cta"] = float(np.max(tr[:, :, 3] - tr[:, :, 0], axis=1).mean()) / mhz
        phases["down_done_max_cta"] = float(np.max(tr[:, rows, 5] - tr[:, rows, 0], axis=1).mean()) / mhz
    tstack.close()
    del layers, routers, biases, xs
    free_device()

    hbm, peak_kind = peaks()
    ffn_bytes = [u * cfg.for_layer(l).expert_bytes() for l, u in enumerate(uniq)]
    expert_bytes_step = sum(ffn_bytes)
    router_bytes_step = cfg.L * cfg.router_bytes()
    step_s = ms / 1e3 / args.steps
    if fused:
        # one persistent kernel per token: it streams every expert and router byte
        kernel = "stack_decode_kernel (fused decode stack, one launch per token)"
        launch_bytes = float(expert_bytes_step + router_bytes_step)
        launch_s = float(route_ms.sum() + ffn_ms.sum()) / 1e3       # the whole kernel
        achieved = launch_bytes / launch_s / 1e9
    else:
        kernel = "ffn_decode_kernel (one launch per layer)"
        launch_bytes = float(statistics.mean(ffn_bytes))
        launch_s = float(ffn_ms.mean()) / 1e3
        achieved = statistics.mean(b / (t / 1e3) for b, t in zip(ffn_bytes, ffn_ms)) / 1e9
    if fused and cfg.fmt_layers:
        traffic = scaled_traffic("stack_decode_mixed", launch_bytes)
    elif fused:
        traffic = stored_traffic("stack_decode") if cfg.L == 48 else None
    else:
        traffic = scaled_traffic("ffn_decode_t8" if cfg.T > 1 else "ffn_decode_t1", launch_bytes)
    out.update({
        "roofline": {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": traffic,
                     "algorithmic_bytes_per_launch": launch_bytes, "avg_launch_us": 1e6 * launch_s,
                     "timing": f"CUDA event nodes around the kernel node(s) of a graph, mean of {n_t} replays"},
        "stack": {"path": "fused persistent kernel" if fused else "per-layer kernels (route + FFN) with PDL",
                  "expert_bytes_per_step": expert_bytes_step, "router_bytes_per_step": router_bytes_step,
                  "expert_GBps": expert_bytes_step / step_s / 1e9,
                  "all_weight_GBps": (expert_bytes_step + router_bytes_step) / step_s / 1e9,
                  "frac_all_weight_of_measured_hbm": (expert_bytes_step + router_bytes_step) / step_s / 1e9 / hbm,
                  "frac_expert_of_8TBps": expert_bytes_step / step_s / 8e12,
                  "route_us_mean": 1e3 * float(route_ms.mean()), "ffn_us_mean": 1e3 * float(ffn_ms.mean()),
                  "fused_phase_us_from_layer_start": phases,
                  "unique_experts_per_layer_mean": statistics.mean(uniq),
                  "reuse_pairs_per_unique_expert": T * cfg.k / statistics.mean(uniq)},
        "e2e": {"value": world * args.steps * T / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * cfg.H * 4, "d2h_bytes_per_step": T * cfg.H * 4,
                "path": "qmoe_stack_decode_host: pinned host x -> graph replay -> pinned host output"},
    })
    return out


def stack_line(args, cfg, m):
    rank, world, _ = dist_env()
    T = cfg.T
    line = {
        "metric": METRIC, "value": m["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": m["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u8 codes x s8 activation limbs -> s32 (tensor core), f32 epilogue, f64 router",
        "data": "synthetic (seeded SplitMix64 weights, Box-Muller activations)",
        "config": dict(workload_desc(cfg, T), parallelism=f"replicas x{world}"),
        "roofline": m["roofline"], "stack": m["stack"], "e2e": m["e2e"], "clocks": m["clocks"],
        "gpu_launches": m["gpu_launches"],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, T)
    return line


def sub_line(line, keep=("value", "unit", "ms_per_step", "config", "roofline", "cpu_baseline", "e2e", "clocks",
                         "gpu_launches", "stack", "prefill", "metric", "route_us_mean")):
    return {k: v for k, v in line.items() if k in keep}


def run_layer(args, cfg):
    """One decode layer per step (router + FFN, one token). The steps cycle
    over LAYER_CYCLE distinct layers whose weights together exceed L2, so every
    step reads its experts from HBM (the kernels' code and small buffers stay
    in L2, as in a decode stack). The step is timed with CUDA events around the
    router and FFN launches (the FFN launch overlaps the router's tail); a
    second pass with an event between them splits the time per kernel."""
    import numpy as np
    import torch

    import quantised_expert_decode_b200 as q
    from synth import gen
    from synth.workload import device_layers

    rank, world, local = dist_env()
    n_layers = LAYER_CYCLE
    layers, routers, _ = device_layers(SEED, cfg, n_layers)
    handles = [l.handle() for l in layers]
    T = cfg.T
    n_in = args.steps + args.warmup
    xs = torch.from_numpy(np.stack([gen.tokens(SEED + 1000 * rank, cfg, i) for i in range(n_in)])).cuda()
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    y = torch.empty((T, cfg.H), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rws = torch.zeros(q.qmoe_route_workspace_bytes(T, cfg.E), dtype=torch.uint8, device="cuda")
    fws = torch.zeros(q.qmoe_decode_workspace_bytes(T, cfg.k, cfg.H, cfg.I), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def step(i, e=None, split=False):
        l = i % n_layers
        if e:
            e[0].record(stream)
        q.qmoe_route(routers[l], None, xs[i], q.F32, T, cfg.H, cfg.E, cfg.k, idx, gate, rws, st, stream)
        if e and split:
            e[1].record(stream)
        q.qmoe_ffn_decode(handles[l], xs[i], T, idx, gate, cfg.k, y, fws, st, stream)
        if e:
            e[2].record(stream)

    def timed(split):
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        barrier(world)
        for i in range(args.steps):
            step(args.warmup + i, ev[i], split)
        torch.cuda.synchronize()
        barrier(world)
        return ev

    clocks = clock_sampler(local)
    ev = timed(False)
    clk = clocks.stop()
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    ev2 = timed(True)
    if q.qmoe_read_status(st) != 0:
        raise RuntimeError("device status set")
    route_ms = [e[0].elapsed_time(e[1]) for e in ev2]
    ffn_ms = [e[1].elapsed_time(e[2]) for e in ev2]
    layer_ms = max_over_ranks(sum(step_ms), world)
    hbm, peak_kind = peaks()
    ffn_bytes = cfg.k * cfg.expert_bytes()
    achieved = ffn_bytes / (statistics.mean(ffn_ms) / 1e3) / 1e9
    weights_mb = n_layers * (cfg.E * cfg.expert_bytes() + cfg.router_bytes()) / 1e6
    line = {"metric": "routed-MoE decode layer tokens/s (one layer); HBM GB/s on expert bytes vs peak",
            "value": replica_throughput(world, args.steps, T, layer_ms), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": layer_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "u8 codes x s8 activation limbs -> s32 (tensor core), f32 epilogue, f64 router",
            "data": "synthetic",
            "config": {"workload": f"one decode layer: {cfg.E} Q{cfg.fmt} experts, hidden {cfg.H}, intermediate "
                                   f"{cfg.I}, top-{cfg.k}, {T} token; steps cycle over {n_layers} distinct seeded "
                                   f"layers ({weights_mb:.0f} MB of weights, larger than L2), no flush; step time = "
                                   f"router + FFN launches, CUDA events around both"},
            "roofline": {"bound": "hbm", "kernel": "ffn_decode_kernel", "achieved": achieved, "peak": hbm,
                         "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                         "traffic": scaled_traffic("ffn_decode_t1", ffn_bytes),
                         "algorithmic_bytes_per_launch": ffn_bytes,
                         "avg_launch_us": 1e3 * statistics.mean(ffn_ms),
                         "median_launch_us": 1e3 * statistics.median(ffn_ms),
                         "timing": "CUDA events around each FFN launch (a second pass, event between router and "
                                   "FFN, so the FFN launch does not overlap the router there)"},
            "route_us_mean": 1e3 * statistics.mean(route_ms), "clocks": clk,
            "gpu_launches": 2 * args.steps}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg, T, n_layers=1, repeats=3)
    del layers, routers, handles, xs
    free_device()
    return line


# ---------------------------------------------------------------- prefill --
def prefill_desc(cfg):
    return {"workload": f"prefill chunk: {cfg.T} bf16 tokens through one {cfg.E}-expert layer, hidden {cfg.H}, "
                        f"intermediate {cfg.I}, top-{cfg.k}, Q{cfg.fmt} blocks, biased router",
            "tokens_per_step": cfg.T, "experts": cfg.E, "hidden": cfg.H, "intermediate": cfg.I, "top_k": cfg.k,
            "format": f"Q{cfg.fmt}", "seed": SEED,
            "l2": "no flush: each step streams the ~1 GB of Q4 weights of its active experts (> 126 MB L2); "
                  "4 distinct activation draws rotate between steps"}


def prefill_flops(cfg, pairs):
    return 2.0 * 3 * cfg.H * cfg.I * pairs, 2.0 * 2 * cfg.H * cfg.I * pairs   # layer, GEMM 1


def oracle_prefill_time(cfg, n_tok):
    """Seconds per token of the float64 oracle: routing of the whole chunk
    (charged per token) plus expert FFNs and combine of n_tok tokens."""
    import numpy as np
    from oracle import moe
    from oracle import workload as W
    x = W.x_float(SEED, cfg)
    Wr, b = gen_router_bias(cfg)
    t0 = time.perf_counter()
    idx, g, _ = moe.route(x, Wr, b, cfg.k)
    t_route = time.perf_counter() - t0
    from synth import gen
    rows = np.arange(n_tok)
    raw = {int(e): gen.expert(SEED, cfg, 0, int(e)) for e in set(idx[rows].ravel().tolist())}
    bits = cfg.format.bits
    t0 = time.perf_counter()

    def get(e):
        r = raw[e]
        return tuple(moe.dequantize(r[n + "_codes"], r[n + "_scales"], bits) for n in ("gate", "up", "down"))
    moe.moe_layer(x[rows], idx[rows], g[rows], get)
    t_ffn = time.perf_counter() - t0
    return t_route / cfg.T + t_ffn / n_tok, t_route, t_ffn


def gen_router_bias(cfg):
    from synth import gen
    return gen.router(SEED, cfg, 0), gen.bias(SEED, cfg, 0)


def run_prefill_reference(args, cfg):
    """The oracle as the reference arm: each step runs it on a bounded sample of
    the chunk (routing of all tokens, FFNs of 8 tokens), scaled per token; at
    most 2 timed steps and 1 warm-up step so the run stays within minutes."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    n_tok, steps, warm = 8, max(1, min(args.steps, 2)), min(args.warmup, 1)
    for _ in range(warm):
        oracle_prefill_time(cfg, n_tok)
    per = [oracle_prefill_time(cfg, n_tok)[0] for _ in range(steps)]
    per_tok = statistics.mean(per)
    value = 1.0 / per_tok
    line = {"impl": "reference", "metric": PREFILL_METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warm, "ms_per_step": 1e3 * per_tok * cfg.T,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": prefill_desc(cfg),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"per step: routing of all {cfg.T} tokens (charged per token) + expert FFNs "
                                       f"and combine of {n_tok} tokens; weight generation excluded"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_prefill(args, cfg):
    import numpy as np
    import torch

    import quantised_expert_decode_b200 as q
    from quantised_expert_decode_b200 import _lib as L
    from synth import gen
    from synth.workload import device_layers

    rank, world, local = dist_env()
    T, k, E, H, I = cfg.T, cfg.k, cfg.E, cfg.H, cfg.I
    layers, routers, biases = device_layers(SEED, cfg, 1)
    layer, Wr, bias = layers[0], routers[0], biases[0]
    n_in = 4
    xs_host = [gen.tokens(SEED + 1000 * rank, cfg, s).view(np.int16) for s in range(n_in)]
    xs = [torch.from_numpy(a).cuda().view(torch.bfloat16) for a in xs_host]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    gate = torch.empty((T, k), dtype=torch.float32, device="cuda")
    y = torch.empty((T, H), dtype=torch.float32, device="cuda")
    rws = torch.zeros(q.qmoe_route_workspace_bytes(T, E), dtype=torch.uint8, device="cuda")
    pws = torch.empty(q.qmoe_prefill_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for es in ev:
        for e in es:
            e.record(stream)
    h = layer.handle()

    def step(s, events=None):
        x = xs[s % n_in]
        q.qmoe_route(Wr, bias, x, L.BF16, T, H, E, k, idx, gate, rws, st, stream)
        if events is None:
            q.qmoe_ffn_prefill(h, x, T, idx, gate, k, y, pws, st, stream)
        else:
            q.qmoe_ffn_prefill_timed(h, x, T, idx, gate, k, y, pws, st, events, stream)

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    if int(st.item()) != 0:
        raise RuntimeError("device status set during warm-up")
    clocks = clock_sampler(local)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = q.qmoe_launch_count()
    e0.record(stream)
    for s in range(args.steps):
        step(args.warmup + s, ev[s])
    e1.record(stream)
    torch.cuda.synchronize()
    launches = q.qmoe_launch_count() - n0
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    clk = clocks.stop()
    if int(st.item()) != 0:
        raise RuntimeError("device status set during the timed run")
    g1_ms = [es[0].elapsed_time(es[1]) for es in ev]
    g2_ms = [es[1].elapsed_time(es[2]) for es in ev]
    value = replica_throughput(world, args.steps, T, ms)

    # the same steps with the earlier combine (fp32 atomic additions into y,
    # not reproducible bit for bit), to record what the slot-ordered combine costs
    ev_a = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for es in ev_a:
        for e in es:
            e.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e4, e5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e4.record(stream)
    for i in range(args.steps):
        x = xs[(args.warmup + i) % n_in]
        q.qmoe_route(Wr, bias, x, L.BF16, T, H, E, k, idx, gate, rws, st, stream)
        q.qmoe_ffn_prefill_timed(h, x, T, idx, gate, k, y, pws, st, ev_a[i], stream, flags=L.PREFILL_ATOMIC_COMBINE)
    e5.record(stream)
    torch.cuda.synchronize()
    ms_atomic = max_over_ranks(e4.elapsed_time(e5), world)
    g2a_ms = [es[1].elapsed_time(es[2]) for es in ev_a]

    # end to end: pinned bf16 x -> device, route + FFN, y -> pinned host
    xh = [torch.from_numpy(a).pin_memory() for a in xs_host]
    yh = torch.empty((T, H), dtype=torch.float32).pin_memory()
    xdev = torch.empty((T, H), dtype=torch.int16, device="cuda")
    torch.cuda.synchronize()
    barrier(world)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for s in range(args.steps):
        xdev.copy_(xh[s % n_in], non_blocking=True)
        xb = xdev.view(torch.bfloat16)
        q.qmoe_route(Wr, bias, xb, L.BF16, T, H, E, k, idx, gate, rws, st, stream)
        q.qmoe_ffn_prefill(h, xb, T, idx, gate, k, y, pws, st, stream)
        yh.copy_(y, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3), world)

    peak, peak_kind = tensor_peak()
    pairs = T * k
    f_layer, f_g1 = prefill_flops(cfg, pairs)
    f_g2 = f_layer - f_g1
    t1, t2 = statistics.mean(g1_ms) / 1e3, statistics.mean(g2_ms) / 1e3
    counts = np.bincount(idx.cpu().numpy().ravel(), minlength=E)
    padded = int(sum((c + 15) // 16 * 16 for c in counts))
    a1 = f_g1 / t1 / 1e12
    line = {
        "metric": PREFILL_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16 x bf16 -> f32 (tcgen05, Q4 weights dequantised in shared memory), f64 router",
        "data": "synthetic (seeded SplitMix64 weights, Box-Muller bf16 activations, N(0,1) router bias)",
        "config": dict(prefill_desc(cfg), parallelism=f"replicas x{world}"),
        "roofline": {"bound": "tensor", "kernel": "pf_gemm_kernel (grouped GEMM 1: gate/up + SiLU*up epilogue)",
                     "achieved": a1, "peak": peak, "peak_kind": peak_kind, "unit": "TFLOP/s", "frac": a1 / peak,
                     "traffic": stored_traffic("pf_gemm1") if cfg.T == 4096 else None,
                     "algorithmic_flops_per_launch": f_g1, "avg_launch_us": 1e6 * t1,
                     "timing": "CUDA events recorded on the launching stream around each GEMM launch"},
        "prefill": {"gemm2_TFLOPs": f_g2 / t2 / 1e12, "gemm2_frac": f_g2 / t2 / 1e12 / peak,
                    "gemm2_us": 1e6 * t2, "ffn_gemms_frac": f_layer / (t1 + t2) / 1e12 / peak,
                    "layer_TFLOPs_per_step": f_layer / (ms / 1e3 / args.steps) / 1e12,
                    "pairs": pairs, "active_experts": int((counts > 0).sum()), "max_expert_load": int(counts.max()),
                    "mma_columns_padded_over_pairs": padded / pairs,
                    "combine": {"kind": "slot-ordered (GEMM 2 writes gate-scaled pair rows, a combine kernel adds "
                                        "each token's rows in slot order): reproducible bit for bit",
                                "ms_per_step": ms / args.steps,
                                "atomic_ms_per_step": ms_atomic / args.steps,
                                "gemm2_us_atomic": 1e3 * statistics.mean(g2a_ms),
                                "cost_vs_atomic": ms / ms_atomic - 1.0}},
        "e2e": {"value": world * args.steps * T / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 4,
                "path": "pinned bf16 x -> device, qmoe_route + qmoe_ffn_prefill, y -> pinned host"},
        "clocks": clk,
        "gpu_launches": launches,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        per_tok, tr, tf = oracle_prefill_time(cfg, 8)
        line["cpu_baseline"] = {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"routing of all {T} tokens ({tr:.1f} s, charged per token) + expert FFNs "
                                          f"and combine of 8 tokens ({tf:.1f} s); weight generation excluded"}
    del layers, routers, biases, xs, pws
    free_device()
    return line


def ngram_oracle_time(nc, n_tok):
    """Seconds the oracle takes to hash ``n_tok`` tokens and dequantise their
    16 rows each (row bytes drawn from the generator beforehand, not timed)."""
    import numpy as np
    from oracle import ngram
    from synth import gen
    ids = gen.ngram_ids(SEED, nc, 0, T=n_tok)
    rows = ngram.rows(SEED, ids, nc.R)
    codes, scales = gen.ngram_rows(SEED, nc, 0, rows.ravel())
    t0 = time.perf_counter()
    r2 = ngram.rows(SEED, ids, nc.R)
    ngram.gather(codes, scales, np.arange(r2.size).reshape(r2.shape))
    return time.perf_counter() - t0


def run_ngram(args, nc):
    """The n-gram row gather over a device-resident table: one launch per
    4096-token chunk, a fresh chunk of ids per step."""
    import numpy as np
    import torch

    import quantised_expert_decode_b200 as q
    from synth import device, gen

    rank, world, local = dist_env()
    T, D, R = nc.T, nc.D, nc.R
    codes, scales = device.ngram_table(SEED, nc)
    n_in = min(args.steps + args.warmup, 16)
    ids_host = [gen.ngram_ids(SEED + 1000 * rank, nc, s) for s in range(n_in)]
    ids = [torch.from_numpy(a).cuda() for a in ids_host]
    out = torch.empty((T, 16, D), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]

    def step(s, events=None):
        if events:
            events[0].record(stream)
        q.qmoe_ngram_gather(ids[s % n_in], T, SEED, codes, scales, R, D, out, None, stream)
        if events:
            events[1].record(stream)

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    clocks = clock_sampler(local)
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = q.qmoe_launch_count()
    e0.record(stream)
    for s in range(args.steps):
        step(args.warmup + s)
    e1.record(stream)
    torch.cuda.synchronize()
    launches = q.qmoe_launch_count() - n0
    barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    clk = clocks.stop()
    # per-launch durations for the roofline (events around each launch)
    for s in range(args.steps):
        step(args.warmup + s, ev[s])
    torch.cuda.synchronize()
    launch_us = 1e3 * statistics.mean(es[0].elapsed_time(es[1]) for es in ev)
    # one decode token: 16 rows, a latency-bound launch
    one = torch.empty((1, 16, D), dtype=torch.float32, device="cuda")
    e6, e7 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e6.record(stream)
    for s in range(args.steps):
        q.qmoe_ngram_gather(ids[s % n_in][:1], 1, SEED, codes, scales, R, D, one, None, stream)
    e7.record(stream)
    torch.cuda.synchronize()
    one_us = 1e3 * e6.elapsed_time(e7) / args.steps
    # end to end: pinned ids -> device, gather, rows -> pinned host
    idh = [torch.from_numpy(a).pin_memory() for a in ids_host]
    outh = torch.empty((T, 16, D), dtype=torch.float32).pin_memory()
    idd = torch.empty((T, 3), dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    barrier(world)
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record(stream)
    for s in range(args.steps):
        idd.copy_(idh[s % n_in], non_blocking=True)
        q.qmoe_ngram_gather(idd, T, SEED, codes, scales, R, D, out, None, stream)
        outh.copy_(out, non_blocking=True)
    e3.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(e2.elapsed_time(e3), world)

    hbm, peak_kind = peaks()
    launch_bytes = T * (12 + 16 * (nc.row_bytes() + 4 * D))
    achieved = launch_bytes / (launch_us / 1e6) / 1e9
    line = {
        "metric": NGRAM_METRIC, "value": replica_throughput(world, args.steps, T, ms), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u8 Q4 codes + fp16 scales -> f32 (exact), u64 hash",
        "data": "synthetic (seeded SplitMix64 table and token ids)",
        "config": {"workload": f"n-gram row gather: {T} tokens x 16 rows of a {R}-row x {D} Q4 table "
                               f"({R * nc.row_bytes() / 1e9:.2f} GB, one layer)",
                   "tokens_per_step": T, "rows": R, "row_elems": D, "vocab": nc.vocab, "seed": SEED,
                   "l2": f"no flush: the table ({R * nc.row_bytes() / 1e6:.0f} MB) is larger than L2 and each "
                         "step draws fresh ids", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": "ngram_gather_kernel", "achieved": achieved, "peak": hbm,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / hbm,
                     "traffic": stored_traffic("ngram_gather") if (T, D, R) == (4096, 256, 1 << 22) else None,
                     "algorithmic_bytes_per_launch": launch_bytes, "avg_launch_us": launch_us,
                     "timing": "CUDA events around each launch on the launching stream"},
        "one_token_us": one_us,
        "e2e": {"value": world * args.steps * T / (ms_e2e / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": T * 12, "d2h_bytes_per_step": T * 16 * D * 4,
                "path": "pinned int32 ids -> device, qmoe_ngram_gather, fp32 rows -> pinned host"},
        "clocks": clk, "gpu_launches": launches,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_tok = T
        t = ngram_oracle_time(nc, n_tok)
        line["cpu_baseline"] = {"value": n_tok / t, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                                "sample": f"hash and 16-row dequantisation of {n_tok} tokens ({t:.2f} s); "
                                          "row bytes drawn beforehand"}
    del codes, scales, out, ids
    free_device()
    return line


def main():
    args = parse()
    from synth import configs
    if args.workload == "ngram":
        rank = dist_env()[0]
        if args.impl == "reference":
            if rank == 0:
                nc = configs.NGRAM
                for _ in range(args.warmup):
                    ngram_oracle_time(nc, nc.T)
                t = sum(ngram_oracle_time(nc, nc.T) for _ in range(args.steps))
                v = args.steps * nc.T / t
                print(json.dumps({"impl": "reference", "metric": NGRAM_METRIC, "value": v, "unit": "tokens/s",
                                  "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                                  "ms_per_step": 1e3 * t / args.steps,
                                  "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                                  "data": "synthetic", "config": {"workload": "n-gram row gather (oracle)"},
                                  "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": blas_threads(),
                                                   "kind": "oracle",
                                                   "sample": f"one {nc.T}-token chunk: hash and 16-row dequantisation"},
                                  "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                                          "d2h_bytes_per_step": 0}}), flush=True)
            return
        _, world, local = dist_env()
        init_dist(local, world)
        line = run_ngram(args, configs.NGRAM)
        if rank == 0:
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    cfg = configs.get(WORKLOADS[args.workload])
    if args.workload == "prefill" and args.tokens:
        cfg = cfg.with_(T=args.tokens)
    if args.workload in ("decode48", "verify48", "mixed48") and args.layers:
        cfg = cfg.with_(L=args.layers)
    if args.workload == "mixed48":
        cfg = configs.mixed(cfg, MIXED_EVERY)
    if args.impl == "reference" and args.workload == "prefill":
        run_prefill_reference(args, cfg)
        return
    if args.impl == "reference":
        run_reference(args, cfg, cfg.T)
        return
    rank, world, local = dist_env()
    init_dist(local, world)
    if args.workload == "prefill":
        line = run_prefill(args, cfg)
    elif args.workload == "layer":
        line = run_layer(args, cfg)
    else:
        line = stack_line(args, cfg, measure_stack(args, cfg))
        if args.workload == "decode48" and not args.headline_only:
            # the headline workload with two more seeds (weights and tokens),
            # then the other workloads, each on freshly generated weights
            line["seeds"] = [{"seed": SEED, "value": line["value"], "ms_per_step": line["ms_per_step"]}]
            for sd in (SEED + 1, SEED + 2):
                m = measure_stack(args, cfg, seed=sd, full=False)
                line["seeds"].append({"seed": sd, "value": m["value"], "ms_per_step": m["ms_per_step"],
                                      "clocks": m["clocks"]})
            line["config1_layer"] = sub_line(run_layer(args, configs.get(1)))
            c3 = configs.get(3)
            line["config3_verify"] = sub_line(stack_line(args, c3, measure_stack(args, c3)))
            line["config4_prefill"] = sub_line(run_prefill(args, configs.get(4)))
            mx = configs.mixed(cfg, MIXED_EVERY)
            line["mixed48_decode"] = sub_line(stack_line(args, mx, measure_stack(args, mx)))
            line["ngram_gather"] = sub_line(run_ngram(args, configs.NGRAM), keep=(
                "metric", "value", "unit", "ms_per_step", "config", "roofline", "cpu_baseline", "e2e", "clocks",
                "gpu_launches", "one_token_us"))
            line["gpu_launches_all_workloads"] = (line["gpu_launches"] + sum(
                line[k_]["gpu_launches"] for k_ in ("config1_layer", "config3_verify", "config4_prefill",
                                                    "mixed48_decode", "ngram_gather")))
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
