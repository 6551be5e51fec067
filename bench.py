#!/usr/bin/env python
"""LatentMoE layer forward throughput on B200 (tokens/s) and roofline fraction.

One step = one latent_moe_forward over the workload's N tokens (every kernel of
the layer).  Default workload: the 0.5b-preset layer (halfb_uniform: N=4096,
d=768, l=384, 16 routed experts top-2, 2 shared, F=768, G=1536, bf16).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the CPU oracle, timed on host cores)

Multi-GPU (torchrun): token-sharded replicas, no data-path collective; each
rank runs its own N tokens, the time is the max over ranks ("scaling": "weak").
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "LatentMoE layer fwd tokens/s on 1 B200; % of bf16 roofline (FLOPs vs HBM)"
L2_FLUSH_BYTES = 256 << 20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# Algorithmic work of each kernel (per launch, full workload): FLOPs or bytes.
def measured_traffic(wl: synth.Workload, tag: str):
    """DRAM bytes per launch of kernel `tag` from the committed ncu capture, or
    None when there is none for this workload or the kernel source changed since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(tag)
    if not rec or rec.get("workload") != wl.name:
        return None
    src = os.path.join(ROOT, rec["source"])
    with open(src, "rb") as f:
        if hashlib.sha256(f.read()).hexdigest() != rec["source_sha256"]:
            return None
    return float(rec["dram_bytes_per_launch"])


def kernel_work(wl: synth.Workload, tag: str):
    N, d, L, R, k, F, S, G = (wl.n_tokens, wl.d, wl.latent, wl.n_routed, wl.top_k, wl.ff_routed,
                              wl.n_shared, wl.ff_shared)
    es = 2 if wl.dtype == "bf16" else 4
    P = N * k
    if tag == "xpass":      # z = W_down x, router logits, shared gate/up + SiTU
        return "tensor", 2.0 * N * d * (L + R + 2 * S * G)
    if tag == "expert_gemm1":
        return "tensor", 2.0 * P * L * 2 * F
    if tag == "expert_gemm2":
        return "tensor", 2.0 * P * F * L
    if tag == "final":      # shared output projection + W_up RMSNorm(u), one accumulator
        return "tensor", 2.0 * N * (S * G + L) * d
    if tag == "combine":    # read k expert rows + ids/probs, write uhat
        return "hbm", float(P * L * es + P * 8 + N * L * es)
    if tag == "dispatch":
        return "hbm", float(P * 4 + P * 8)
    if tag == "route":
        return "hbm", float(N * d * es + R * d * es + P * 8)
    raise KeyError(tag)


class ClockSampler:
    """Samples the SM clock and the clock-event (throttle) reasons with NVML
    while a region runs, as fast as NVML answers (a sample every ~0.1 ms)."""

    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
               "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
               "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
               "display_clock_setting": 0x100}

    def __init__(self, index: int, period_s: float = 5e-5):
        self.index = index
        self.period_s = period_s
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False

    def _sample(self):
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period_s)

    def start(self):
        if self.ok:
            self._sample()                       # at least one sample, taken at the start
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()
            self._sample()                       # and one at the end
        names = [n for n, bit in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def pick_tensor_peak(peaks: dict, region_s: float, clk: dict):
    """Denominator for a tensor-core kernel: the burst peak (cuBLAS timed alone)
    when the timed region is short (< 1 s) or the SM clock stayed within 2 % of
    its maximum; the sustained (power-capped) peak only for long regions that
    ran at a lower clock."""
    mhz, mx = clk.get("sm_mhz"), clk.get("sm_max_mhz")
    at_max = mhz is not None and mx and mhz >= 0.98 * mx
    if region_s < 1.0 or at_max:
        why = "timed region %.3f s" % region_s if region_s < 1.0 else "SM clock within 2%% of max"
        return peaks["bf16_tflops"], f"{peaks['source']} burst ({why})"
    return peaks["bf16_tflops_sustained"], f"{peaks['source']} sustained (region {region_s:.1f} s)"


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_token_rows(wl: synth.Workload, rank: int) -> np.ndarray:
    """Token rows of one replica: rank r draws x rows [r*N, (r+1)*N) of the stream."""
    return np.arange(wl.n_tokens, dtype=np.int64) + rank * wl.n_tokens


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank number over the process group (the value itself at N = 1)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def cpu_model() -> str:
    """The host CPU's model name (first 'model name' line of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(wl: synth.Workload, seed: int, budget_s: float = 12.0) -> dict:
    """The oracle as it stands on the host cores, on a bounded sample of the
    workload's tokens: first a small probe, then a sample sized to ~budget_s."""
    import oracle
    inp = synth.make_inputs(wl.with_tokens(0), seed, with_x=False)
    w = {k: synth.to_f32(inp[k]) for k in synth.WEIGHT_NAMES}
    cores = os.cpu_count() or 1

    def run(n):
        x = synth.to_f32(synth.make_x_rows(wl, seed, np.arange(n)))
        dims = oracle.Dims(n, wl.d, wl.latent, wl.n_routed, wl.top_k, wl.n_shared, wl.ff_routed,
                           wl.ff_shared, wl.beta1, wl.beta2, wl.rms_eps)
        t0 = time.perf_counter()
        oracle.forward(dims, w, x)
        return time.perf_counter() - t0

    probe_n = max(1, min(wl.n_tokens, cores * 2))
    t_probe = run(probe_n)
    n = int(min(wl.n_tokens, max(probe_n, probe_n * budget_s / max(t_probe, 1e-6))))
    t = run(n)
    return {"value": n / t, "unit": "tokens/s", "cores": int(os.environ.get("OMP_NUM_THREADS", cores)),
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"{n} of {wl.n_tokens} tokens of {wl.name}, fp64 C oracle, OpenMP over tokens, "
                      f"{t:.1f} s"}


def workload_config(wl: synth.Workload, world: int) -> dict:
    """The layer's sizes, shared by both arms' JSON lines."""
    return {"workload": wl.name, "n_tokens": wl.n_tokens, "d": wl.d, "latent": wl.latent,
            "n_routed": wl.n_routed, "top_k": wl.top_k, "ff_routed": wl.ff_routed,
            "n_shared": wl.n_shared, "ff_shared": wl.ff_shared, "parallelism": f"replicas{world}"}


def run_reference(args, wl):
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    import oracle
    inp = synth.make_inputs(wl.with_tokens(0), args.seed, with_x=False)
    w = {k: synth.to_f32(inp[k]) for k in synth.WEIGHT_NAMES}
    cores = os.cpu_count() or 1
    # each step: a bounded sample of the workload's tokens
    probe = max(1, min(wl.n_tokens, cores))
    dims = lambda n: oracle.Dims(n, wl.d, wl.latent, wl.n_routed, wl.top_k, wl.n_shared,
                                 wl.ff_routed, wl.ff_shared, wl.beta1, wl.beta2, wl.rms_eps)
    xp = synth.to_f32(synth.make_x_rows(wl, args.seed, np.arange(probe)))
    t0 = time.perf_counter()
    oracle.forward(dims(probe), w, xp)
    per_tok = (time.perf_counter() - t0) / probe
    total_budget = 60.0
    n_step = int(max(1, min(wl.n_tokens, total_budget / (args.steps + args.warmup) / per_tok)))
    x = synth.to_f32(synth.make_x_rows(wl, args.seed, np.arange(n_step)))
    for _ in range(args.warmup):
        oracle.forward(dims(n_step), w, x)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.forward(dims(n_step), w, x)
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = n_step / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": f"{n_step} of {wl.n_tokens} tokens per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_library_gemm_shapes(args, wl):
    """Context for the roofline: cuBLAS (torch.matmul, bf16, fp32 accumulation)
    on plain GEMMs of the layer's two dense shapes -- the x-pass [N, d] x
    [d, l + R + 2 S G] and the final GEMM [N, S G + l] x [S G + l, d] -- and
    on an 8192^3 square, timed like the forward (CUDA events, L2 flushed
    before each call).  None of this is on the product path."""
    import torch
    dev = torch.device("cuda", 0)
    N, d, L, R, S, G = wl.n_tokens, wl.d, wl.latent, wl.n_routed, wl.n_shared, wl.ff_shared
    shapes = {"xpass": (N, d, L + R + 2 * S * G), "final": (N, S * G + L, d),
              "square": (8192, 8192, 8192)}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    out = {"workload": wl.name, "what": "cuBLAS bf16 plain GEMM [M,K] x [K,N], us and TFLOP/s"}
    for name, (M, K, Nn) in shapes.items():
        a = torch.randn(M, K, device=dev, dtype=torch.bfloat16)
        b = torch.randn(Nn, K, device=dev, dtype=torch.bfloat16)
        for _ in range(max(3, args.warmup)):
            a @ b.t()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            a @ b.t()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        us = total / args.steps * 1e3
        out[name] = {"M": M, "K": K, "N": Nn, "us": round(us, 2),
                     "tflops": round(2.0 * M * K * Nn / (us * 1e-6) / 1e12, 1)}
    print(json.dumps(out))
    return 0


def run_memory_kernels(args, wl):
    """Routing, dispatch and combine called on their own through the C ABI at the
    workload's shapes (synthetic activations; no expert weights), each timed with
    CUDA events over --steps calls with L2 flushed in between.  Prints one JSON
    line per entry point: algorithmic bytes per call (what the entry point must read and write),
    time, and the fraction of the roof max(bytes / HBM, FLOPs / bf16 peak)."""
    import torch
    import sigmoid_top_routing_latentmoe_b200 as lm
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(args.seed)
    N, d, L, R, k = wl.n_tokens, wl.d, wl.latent, wl.n_routed, wl.top_k
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    es = 2 if wl.dtype == "bf16" else 4
    P = N * k
    dims = lm.make_dims(N, d, L, R, k, 0, wl.ff_routed, wl.ff_routed, wl.beta1, wl.beta2,
                        wl.rms_eps, dt)
    ws = lm.alloc_workspace(dims)
    x = torch.randn(N, d, generator=g, device="cuda").to(dt)
    w_r = (torch.randn(R, d, generator=g, device="cuda") * 0.02).to(dt)
    ids = torch.empty(N, k, dtype=torch.int32, device="cuda")
    probs = torch.empty(N, k, dtype=torch.float32, device="cuda")
    counts = torch.empty(R, dtype=torch.int32, device="cuda")
    offs = torch.empty(R + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(P, dtype=torch.int32, device="cuda")
    inv = torch.empty(P, dtype=torch.int32, device="cuda")
    eo = torch.randn(P, L, generator=g, device="cuda").to(dt)
    rms_w = torch.ones(L, dtype=torch.float32, device="cuda")
    u = torch.empty(N, L, dtype=dt, device="cuda")
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    calls = {
        "route": (lambda: lm.moe_route(dims, x, w_r, None, ids, probs, ws),
                  N * d * es + R * d * es + P * 8, 2.0 * N * d * R),
        "dispatch": (lambda: lm.moe_dispatch(dims, ids, counts, offs, perm, inv, ws),
                     P * 4 + P * 8, 0.0),
        "combine": (lambda: lm.moe_combine(dims, eo, inv, probs, rms_w, u),
                    P * L * es + P * 8 + N * L * es, 0.0),
    }
    peaks = _peaks()
    for name, (fn, nbytes, flops) in calls.items():
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        total = 0.0
        for _ in range(args.steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        us = total / args.steps * 1e3
        roof_us = max(nbytes / (peaks["hbm_gbs"] * 1e3), flops / (peaks["bf16_tflops"] * 1e6))
        print(json.dumps({"kernel": name, "workload": wl.name, "us": us, "bytes": nbytes,
                          "flops": flops, "gb_s": nbytes / us / 1e3,
                          "hbm_frac": nbytes / us / 1e3 / peaks["hbm_gbs"],
                          "roof_us": roof_us, "roof_frac": roof_us / us,
                          "note": ("includes the router-logit GEMM on the tensor cores"
                                   if R > 32 else "router GEMV on the CUDA cores"
                                   ) if name == "route" else ""}), flush=True)
    if lm.get_device_status(ws) != lm.OK:
        raise SystemExit("device status not OK")


# fp32 FFMA peak of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz (max SM clock)
FP32_SIMT_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_backward_bench(args, wl):
    """latent_moe_backward timed like the forward (CUDA graph replay, L2 flushed
    between steps); one JSON line.  Algorithmic work: the gradient contractions,
    2x the forward's FLOPs (the backward also recomputes the forward, 1x more),
    on the CUDA cores in fp32."""
    import torch
    import sigmoid_top_routing_latentmoe_b200 as lm
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    inp = synth.make_inputs(wl, args.seed)

    def todev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    w = {k: todev(inp[k]) for k in synth.WEIGHT_NAMES}
    x = todev(inp["x"])
    dy = todev(synth.normal(args.seed + 1, "dy", (wl.n_tokens, wl.d), 1.0,
                            dtype="bf16" if wl.dtype == "bf16" else "f32"))
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dims = lm.make_dims(wl.n_tokens, wl.d, wl.latent, wl.n_routed, wl.top_k, wl.n_shared,
                        wl.ff_routed, wl.ff_shared, wl.beta1, wl.beta2, wl.rms_eps, dt)
    ws = lm.alloc_backward_workspace(dims, device=dev)
    N, d, L, R, F, S, G = (wl.n_tokens, wl.d, wl.latent, wl.n_routed, wl.ff_routed, wl.n_shared,
                           wl.ff_shared)
    shapes = {"dx": (N, d), "dw_down": (L, d), "dw_router": (R, d), "dw_up": (d, L),
              "drms_weight": (L,), "dw_g": (R, F, L), "dw_u": (R, F, L), "dw_o": (R, L, F)}
    if S:
        shapes.update(dws_g=(S, G, d), dws_u=(S, G, d), dws_o=(S, d, G))
    grads = {n: torch.empty(sh, dtype=torch.float32, device=dev) for n, sh in shapes.items()}
    wstruct = lm.weights_struct(w)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        lm.latent_moe_backward(dims, wstruct, x, dy, grads, ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if lm.get_device_status(ws) != lm.OK:
        raise SystemExit("device status not OK after warm-up")
    lm.launch_count(reset=True)
    graph = torch.cuda.CUDAGraph()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.graph(graph, stream=cap):
        step()
    launches = lm.launch_count(reset=True)
    graph.replay()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    stream = torch.cuda.current_stream(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    clocks.start()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        graph.replay()
        ends[i].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    work = 2.0 * wl.flops()
    achieved = work / (ms / 1e3) / 1e12
    print(json.dumps({
        "metric": "LatentMoE layer bwd tokens/s on 1 B200 (gradients of x and every weight)",
        "value": wl.n_tokens / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (from %s inputs)" % wl.dtype, "data": "synthetic",
        "config": {"workload": wl.name, "n_tokens": wl.n_tokens, "launch": "cuda graph replay",
                   "l2": "flushed (256 MiB write) between steps"},
        "roofline": {"kernel": "whole backward", "bound": "alu", "achieved": achieved,
                     "peak": FP32_SIMT_TFLOPS, "unit": "TFLOP/s",
                     "frac": achieved / FP32_SIMT_TFLOPS, "traffic": None,
                     "work": "2x forward FLOPs (the recomputed forward is not counted)"},
        "clocks": clk, "gpu_launches": launches * args.steps}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="halfb_uniform", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--profile-kernel", default=None,
                    help="kernel tag for the roofline line (default: the largest GEMM)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true",
                    help="launch the kernels every step instead of replaying a CUDA graph")
    ap.add_argument("--memory-kernels", action="store_true",
                    help="time moe_route / moe_dispatch / moe_combine on their own instead")
    ap.add_argument("--backward", action="store_true",
                    help="time latent_moe_backward instead of the forward")
    ap.add_argument("--library-gemm-shapes", action="store_true",
                    help="time cuBLAS on plain GEMMs of the layer's dense shapes (context only)")
    ap.add_argument("--sustained-seconds", type=float, default=1.0,
                    help="length of the back-to-back replay pass whose clocks are reported as "
                         "clocks_sustained (0: no such pass, e.g. under a profiler)")
    args = ap.parse_args()
    wl = synth.WORKLOADS[args.workload]
    if args.memory_kernels:
        return run_memory_kernels(args, wl)
    if args.library_gemm_shapes:
        return run_library_gemm_shapes(args, wl)
    if args.backward:
        return run_backward_bench(args, wl)
    if args.impl == "reference":
        return run_reference(args, wl)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    import torch
    import torch.distributed as dist

    import sigmoid_top_routing_latentmoe_b200 as lm

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    # inputs: weights shared by all ranks (seed), x drawn per rank (its own tokens)
    inp = synth.make_inputs(wl, args.seed, with_x=False)
    x_np = synth.make_x_rows(wl, args.seed, rank_token_rows(wl, rank))

    def todev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    w = {k: todev(inp[k]) for k in synth.WEIGHT_NAMES}
    x = todev(x_np)
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    dims = lm.make_dims(wl.n_tokens, wl.d, wl.latent, wl.n_routed, wl.top_k, wl.n_shared,
                        wl.ff_routed, wl.ff_shared, wl.beta1, wl.beta2, wl.rms_eps, dt)
    ws = lm.alloc_workspace(dims, device=dev)
    y = torch.empty(wl.n_tokens, wl.d, dtype=dt, device=dev)
    wstruct = lm.weights_struct(w)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step():
        lm.latent_moe_forward(dims, wstruct, x, y, ws)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if lm.get_device_status(ws) != lm.OK:
        raise SystemExit("device status not OK after warm-up")

    prof_tag = args.profile_kernel or "xpass"
    plan = lm.forward_plan(dims)
    bound, work = kernel_work(wl, prof_tag)
    lm.profile_read()                       # drop anything recorded so far
    clocks = ClockSampler(local)

    # One step is captured once in a CUDA graph (with the dominant kernel
    # bracketed by events) and replayed; --eager launches it every step.
    graph = None
    launches_per_step = None
    if not args.eager:
        lm.launch_count(reset=True)
        lm.profile_enable(prof_tag)
        graph = torch.cuda.CUDAGraph()
        cap_stream = torch.cuda.Stream(dev)
        cap_stream.wait_stream(stream)
        with torch.cuda.graph(graph, stream=cap_stream):
            step()
        lm.profile_enable(None)
        launches_per_step = lm.launch_count(reset=True)
        graph.replay()
        torch.cuda.synchronize()
    else:
        lm.profile_enable(prof_tag)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    lm.launch_count(reset=True)
    k_ms, k_n = 0.0, 0
    region0 = torch.cuda.Event(enable_timing=True)
    region1 = torch.cuda.Event(enable_timing=True)
    clocks.start()
    region0.record(stream)
    for i in range(args.steps):
        flush.zero_()                        # L2 flushed between timed steps (outside the events)
        starts[i].record(stream)
        if graph is not None:
            graph.replay()
        else:
            step()
        ends[i].record(stream)
        if graph is not None:                # the graph re-records its events on every replay
            ms_i, n_i = lm.profile_peek(prof_tag)
            k_ms += ms_i
            k_n += n_i
    region1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    region_s = region0.elapsed_time(region1) / 1e3
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms_per_step = max_over_ranks(float(sum(step_ms)), dev) / args.steps

    if graph is None:                        # eager: the timed region's own launches and events
        launches = lm.launch_count()
        lm.profile_enable(None)
        k_ms, k_n = lm.profile_read(prof_tag)
    # (both passes replay the graph, whose event-record nodes use the profiling
    # events: they run before lm.profile_read() releases those events)
    # hot: the same K steps back to back, L2 not flushed (weights and x stay cached)
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    h0.record(stream)
    for _ in range(args.steps):
        graph.replay() if graph is not None else step()
    h1.record(stream)
    torch.cuda.synchronize()
    hot_ms = max_over_ranks(h0.elapsed_time(h1) / args.steps, dev)
    # sustained clocks: >= 1 s of back-to-back replays, sampled like the timed region
    n_sus = int(math.ceil(args.sustained_seconds / max(ms_per_step / 1e3, 1e-6)))
    sus = ClockSampler(local)
    if world > 1:
        dist.barrier()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sus.start()
    s0.record(stream)
    for _ in range(n_sus):
        graph.replay() if graph is not None else step()
    s1.record(stream)
    torch.cuda.synchronize()
    clk_sus = sus.stop()
    clk_sus["seconds"] = s0.elapsed_time(s1) / 1e3
    clk_sus["steps"] = n_sus
    clk_sus["ms_per_step"] = s0.elapsed_time(s1) / n_sus if n_sus else None
    if graph is not None:
        launches = launches_per_step * args.steps
        lm.profile_read()
    value = world * wl.n_tokens / (ms_per_step / 1e3)
    if lm.get_device_status(ws) != lm.OK:
        raise SystemExit("device status not OK after the timed region")


    # per-kernel breakdown (a separate pass with every kernel bracketed by events)
    lm.profile_enable("*")
    for _ in range(min(args.steps, 20)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    lm.profile_enable(None)
    breakdown = {}
    for tag in ("xpass", "route", "dispatch", "gather", "expert_gemm1", "expert_gemm2", "combine",
                "final"):
        ms, n = lm.profile_read(tag)
        if n:
            breakdown[tag] = round(ms / min(args.steps, 20) * 1e3, 2)
    lm.profile_read()

    # host time to enqueue one eager forward (the call returns once everything is queued)
    enq = []
    for _ in range(5):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        step()
        enq.append(time.perf_counter() - t0)
    torch.cuda.synchronize()
    host_enqueue_us = statistics.median(enq) * 1e6

    # end to end through the host entry point: pinned x in, y out, copies timed
    ws_h = lm.alloc_workspace(dims, device=dev, host=True)
    x_h = x.cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    for _ in range(3):
        lm.latent_moe_forward_host(dims, wstruct, x_h, y_h, ws_h)
    e2e_steps = max(3, min(args.steps, 50))
    if world > 1:
        dist.barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(e2e_steps):
        lm.latent_moe_forward_host(dims, wstruct, x_h, y_h, ws_h)
    ev1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps, dev)
    io_bytes = wl.n_tokens * wl.d * (2 if wl.dtype == "bf16" else 4)
    # the copies alone: x in and y out through the same pinned buffers, on two
    # streams at once (what the host link allows per step, with no compute)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    x_d, y_d = torch.empty_like(x), torch.empty_like(x)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for it in range(e2e_steps + 3):
        if it == 3:
            c0.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        with torch.cuda.stream(s_in):
            x_d.copy_(x_h, non_blocking=True)
        with torch.cuda.stream(s_out):
            y_h.copy_(y_d, non_blocking=True)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
    c1.record(stream)
    torch.cuda.synchronize()
    copy_ms = c0.elapsed_time(c1) / e2e_steps

    peaks = _peaks()
    if k_n > 0:
        k_avg_s = k_ms / k_n / 1e3
        if bound == "tensor":
            achieved = work / k_avg_s / 1e12
            peak, peak_source = pick_tensor_peak(peaks, region_s, clk)
            unit = "TFLOP/s"
        else:
            achieved = work / k_avg_s / 1e9
            peak, peak_source = peaks["hbm_gbs"], peaks["source"]
            unit = "GB/s"
        roof = {"kernel": prof_tag, "bound": bound, "achieved": achieved, "peak": peak,
                "unit": unit, "frac": achieved / peak, "traffic": measured_traffic(wl, prof_tag),
                "launch_us": k_avg_s * 1e6, "launches": k_n, "peak_source": peak_source}
    else:
        roof = None
    # bytes the layer must read: the weights of the experts this input routes to
    counts = torch.zeros(wl.n_routed, dtype=torch.int32, device=dev)
    lm.latent_moe_forward(dims, wstruct, x, y, ws, counts_out=counts)
    used = int((counts > 0).sum().item())
    cbytes = wl.compulsory_bytes(used)
    roof_s = max(wl.flops() / (peaks["bf16_tflops"] * 1e12), cbytes / (peaks["hbm_gbs"] * 1e9))
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": wl.dtype, "data": "synthetic",
        "config": dict(workload_config(wl, world), l2="flushed (256 MiB write) between steps",
                       launch="eager" if args.eager else "cuda graph replay"),
        "layer_roofline": {"flops": wl.flops(), "compulsory_bytes": cbytes, "experts_used": used,
                           "roof_us": roof_s * 1e6, "frac": roof_s / (ms_per_step / 1e3),
                           "peak_source": peaks["source"] + " burst"},
        "roofline": roof,
        "clocks": dict(clk, region_s=region_s),
        "clocks_sustained": clk_sus,
        "hot": {"value": world * wl.n_tokens / (hot_ms / 1e3), "unit": "tokens/s",
                "ms_per_step": hot_ms, "l2": "not flushed (back-to-back steps)"},
        "e2e": {"value": world * wl.n_tokens / (e2e_ms / 1e3), "unit": "tokens/s",
                "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes,
                "ms_per_step": e2e_ms,
                "copies_alone_ms_per_step": copy_ms,
                "copy_bound": world * wl.n_tokens / (copy_ms / 1e3)},
        "gpu_launches": launches,
        "host_enqueue_us": host_enqueue_us,
        "kernel_us": breakdown,
        "plan": [name for name, on in plan.items() if on],
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.seed)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
