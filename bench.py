"""Benchmark of the W4A4 ConvRot linear layer on B200.

Workload (default): the Flux-like attention projection, M = 4608 tokens (4096
image + 512 text), K = N = 3072, ConvRot group 128, bias, no low-rank branch.
One step = one whole layer over one batch: rotate + quantize the bf16
activations (K1), then the INT4 GEMM with the fused dequant + bias epilogue
(K2) -- the same two launches w4a4_linear makes.  Inputs are synthetic
(seeded NumPy draws in the shape and value mix of the pages' workload) and
resident in HBM; four input sets (about 272 MB) rotate so that no step finds
its inputs in the 126 MB L2.  The K timed steps are captured once as a CUDA
graph of layer calls and replayed (the launch pattern of a server running
fixed-shape layers); the same K calls launched one by one from the host are
reported beside it.

Prints one JSON line (rank 0).  Metric: TOPS = 2 M N K / time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs one independent layer per GPU (weak scaling: the path shards by
tokens with no exchange), timed on the device, max over ranks.
--impl reference times the CPU oracle on the host cores on a bounded sample
of the same workload.
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

INT8_NOMINAL_TOPS = 4500.0     # B200 dense INT8 tensor peak (datasheet)
HBM_NOMINAL_GBS = 8000.0
# measured on this part: one pair MMA M256 N256 K32 int8 every 128 cycles
# = 8192 int8 MAC per clock per SM; the clock-adjusted peak uses it with the
# SM clock sampled during the run
INT8_MAC_PER_CLK_PER_SM = 8192


def clock_adjusted_peak_tops(sm_mhz, sms: int = 148):
    if not sm_mhz:
        return None
    return 2.0 * INT8_MAC_PER_CLK_PER_SM * sms * sm_mhz * 1e6 / 1e12

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# the ncu captures summarised in profiles/, valid only for the kernel code they
# were taken from: keyed by a hash of the source file with its comments and
# whitespace removed (so an edited comment keeps the figure, any code change
# drops it to null).
MEASURED_TRAFFIC = {
    ("gemm", "attn_proj"): ("w4a4_int4_quantized_b200/csrc/gemm.cu", "2109f93cdeed1d86", 11.892e6),
    ("gemm", "m256_down"): ("w4a4_int4_quantized_b200/csrc/gemm.cu", "2109f93cdeed1d86", 20.503e6),
    ("gemm_w4a8", "attn_proj"): ("w4a4_int4_quantized_b200/csrc/gemm.cu", "2109f93cdeed1d86", 19.174e6),
    ("rotate_quantize", "attn_proj"): ("w4a4_int4_quantized_b200/csrc/quantize.cu", "003946100a4d56c2", 28.378e6),
}


def code_hash(text: str) -> str:
    """sha256 prefix of C/C++/CUDA source with comments and whitespace removed."""
    import hashlib
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return hashlib.sha256(" ".join(text.split()).encode()).hexdigest()[:16]


def _traffic(kernel: str, workload: str):
    if (kernel, workload) not in MEASURED_TRAFFIC:
        return None
    path, sha, value = MEASURED_TRAFFIC[(kernel, workload)]
    try:
        with open(os.path.join(ROOT, path)) as f:
            cur = code_hash(f.read())
    except OSError:
        return None
    return value if cur == sha else None


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region.

    Samples are time-stamped on arrival; `stop` keeps those that fall inside
    the marked window (plus the first one after it, which covers the window's
    end), so a short timed region still reports the clocks it ran at."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, interval_ms: int = 20):
        self.index = index
        self.interval_ms = interval_ms
        self.proc = None
        self.lines: list[tuple[float, str]] = []
        self.window = (0.0, float("inf"))

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.interval_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.perf_counter(), line.strip()))

    def mark(self, t0: float, t1: float):
        self.window = (t0, t1)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(2 * self.interval_ms / 1e3)   # let the sample after the window arrive
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self._t.join(timeout=2)
        t0, t1 = self.window
        inside = [ln for t, ln in self.lines if t0 <= t <= t1]
        after = [ln for t, ln in self.lines if t > t1][:1]
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in inside + after:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "window_ms": round((t1 - t0) * 1e3, 2) if t1 != float("inf") else None}


def _dist_init(n_gpus: int):
    from w4a4_int4_quantized_b200.shard import dist_env
    rank, world, local = dist_env()
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return rank, world, local


def cpu_baseline(spec, budget_s: float = 10.0, variant: str = "w4a4") -> dict:
    """The CPU oracle as it stands, on the host cores, on a bounded sample of
    the workload: the per-step path (activation rotate + quantize, integer
    GEMM, epilogue) for a subset of token rows against the full weight matrix
    (weights are quantized once, offline, as on the GPU)."""
    import oracle
    from w4a4_int4_quantized_b200 import inputs
    d = inputs.make_layer(spec)
    if variant == "w4a8":
        _, ws, wz, wu = oracle.quantize_w4a8_weights(d["W"], spec.group)
        wq = (wu.astype(np.int16) - wz.astype(np.int16)[:, None]).astype(np.int8)
    else:
        _, ws, wq = oracle.quantize_w4(d["W"], spec.group)
    rows = 8
    while True:
        t0 = time.perf_counter()
        if variant == "w4a8":
            xq, xs = oracle.quantize_w8(d["X"][:rows], spec.group)
        else:
            _, xs, xq = oracle.quantize_w4(d["X"][:rows], spec.group)
        acc = oracle.int_gemm(xq, wq)
        oracle.epilogue(acc, xs, ws, spec.group, None, None, d["bias"])
        dt = time.perf_counter() - t0
        if dt >= budget_s or rows >= spec.M:
            break
        rows = min(spec.M, max(rows * 2, int(rows * budget_s / max(dt, 1e-3) * 1.1)))
    ops = 2.0 * rows * spec.N * spec.K
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{rows} of {spec.M} token rows x full {spec.N}x{spec.K} weights "
                      f"(act quant + int GEMM + epilogue), {dt:.1f} s"}


def _metric_name(variant: str, spec) -> str:
    v = variant.upper()
    return (f"{v} linear TOPS & us/layer (M={spec.M},K={spec.K},N={spec.N}) and % of B200 INT8 TC peak"
            if spec.name != "attn_proj" or variant != "w4a4"
            else "W4A4 linear TOPS & us/layer (M=4608,K=N=3072) and % of B200 INT8 TC peak")


def run_reference(args, spec):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(spec, budget_s=budget / 4, variant=args.variant)
    vals = [cpu_baseline(spec, budget_s=budget, variant=args.variant) for _ in range(args.steps)]
    v = statistics.median([b["value"] for b in vals])
    line = {
        "impl": "reference", "metric": _metric_name(args.variant, spec), "value": v, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 2.0 * spec.M * spec.N * spec.K / (v * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("int8 x 4-bit" if args.variant == "w4a8" else "int4") + " codes, int64 acc, f64 epilogue",
        "data": "synthetic", "config": {"workload": spec.name, "M": spec.M, "K": spec.K, "N": spec.N,
                                        "group": spec.group, "rank": spec.rank},
        "cpu_baseline": {"value": v, "unit": "TOPS", "cores": vals[0]["cores"], "kind": "oracle",
                         "sample": vals[0]["sample"]},
        "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_mlp(args):
    """The MLP pair at M = 4608 (3072 -> 12288 -> 3072, r = 128 on both, g = 128)
    with GELU fused into the up-projection epilogue: per step rotate+quantize
    X, low-rank down, up GEMM with GELU, rotate+quantize h, low-rank down,
    down GEMM.  Also times the unfused chain (plain up GEMM, torch GELU on
    [M, 12288] bf16, same down layer) for comparison.  Single GPU."""
    import torch
    import w4a4_int4_quantized_b200 as w4
    from w4a4_int4_quantized_b200 import inputs
    w4.load_library()
    su, sd = inputs.WORKLOADS["mlp_up"], inputs.WORKLOADS["mlp_down"]
    M, D, H, g, r = su.M, su.K, su.N, su.group, su.rank

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    du, dd = inputs.make_layer(su), inputs.make_layer(sd)
    Wq_u, ws_u = w4.w4a4_quantize_weights(dev(du["W"]), g)
    Wq_d, ws_d = w4.w4a4_quantize_weights(dev(dd["W"]), g)
    L1u, L2u, bu = dev(du["L1"]), dev(du["L2"]), dev(du["bias"])
    L1d, L2d, bd = dev(dd["L1"]), dev(dd["L2"]), dev(dd["bias"])
    sets = []
    for i in range(2):
        X = dev(inputs.make_layer(su, seed_offset=i)["X"])
        sets.append(dict(X=X, Xq=torch.empty((M, D // 2), dtype=torch.uint8, device="cuda"),
                         xs=torch.empty((M,), dtype=torch.float32, device="cuda"),
                         T=torch.empty((M, r), dtype=torch.bfloat16, device="cuda"),
                         h=torch.empty((M, H), dtype=torch.bfloat16, device="cuda"),
                         hq=torch.empty((M, H // 2), dtype=torch.uint8, device="cuda"),
                         hs=torch.empty((M,), dtype=torch.float32, device="cuda"),
                         Th=torch.empty((M, r), dtype=torch.bfloat16, device="cuda"),
                         Y=torch.empty((M, D), dtype=torch.bfloat16, device="cuda")))
    def step(s, fused=True):
        stream = torch.cuda.current_stream()
        w4.w4a4_rotate_quantize_act(s["X"], g, L1u, Xq=s["Xq"], x_scale=s["xs"], T=s["T"], stream=stream)
        if fused:
            w4.w4a4_gemm_gelu(s["Xq"], s["xs"], Wq_u, ws_u, g, s["T"], L2u, bu, Y=s["h"], stream=stream)
        else:
            w4.w4a4_gemm(s["Xq"], s["xs"], Wq_u, ws_u, g, s["T"], L2u, bu, Y=s["h"], stream=stream)
            s["h"].copy_(torch.nn.functional.gelu(s["h"], approximate="tanh"))
        w4.w4a4_rotate_quantize_act(s["h"], g, L1d, Xq=s["hq"], x_scale=s["hs"], T=s["Th"], stream=stream)
        w4.w4a4_gemm(s["hq"], s["hs"], Wq_d, ws_d, g, s["Th"], L2d, bd, Y=s["Y"], stream=stream)

    def timed(fused, n):
        # n steps captured in a CUDA graph and replayed
        for i in range(args.warmup):
            step(sets[i % 2], fused)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            for i in range(n):
                step(sets[i % 2], fused)
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        del graph
        return e0.elapsed_time(e1) / n

    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    t0 = time.perf_counter()
    ms = timed(True, args.steps)
    clocks.mark(t0, time.perf_counter())
    clk = clocks.stop()
    ms_unfused = timed(False, args.steps)
    err = w4.w4a4_get_device_error()
    if err:
        raise SystemExit(f"device error word {err:#x}")
    ops = 2.0 * 2.0 * M * D * H
    lr_flops = 2.0 * 2.0 * M * r * (D + H)
    pk = _peaks()
    line = {
        "metric": "W4A4 fused MLP pair TOPS & us (M=4608, 3072->12288->3072, r=128, GELU in the up epilogue)",
        "value": ops / (ms * 1e-3) / 1e12, "unit": "TOPS", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "us_per_mlp": ms * 1e3, "us_per_mlp_unfused": ms_unfused * 1e3,
        "lowrank_gflop_per_step": lr_flops / 1e9,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 codes (int8 MMA, int32 acc), bf16 in/out", "data": "synthetic",
        "config": {"workload": "mlp_pair", "M": M, "D": D, "H": H, "group": g, "rank": r,
                   "l2": "2 rotating input sets; [M, 12288] intermediates exceed L2"},
        "roofline": {"bound": "tensor", "achieved": ops / (ms * 1e-3) / 1e12, "peak": 2.0 * pk["bf16"],
                     "unit": "TOPS", "frac": ops / (ms * 1e-3) / 1e12 / (2.0 * pk["bf16"]),
                     "traffic": None, "peak_note": "whole chain against the int8 tensor peak (2 x burst bf16)"},
        "gpu_launches": 6 * args.steps, "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def run_bake(args):
    """Baking a LoRA of rank --bake-lora into the attention-projection weights
    (N = K = 3072, g = 128) and re-quantizing them with stochastic rounding:
    the fp32 bake kernel and the stochastic-rounding rotate + quantize, per
    call.  An offline step (once per LoRA change), reported as time."""
    import torch
    import w4a4_int4_quantized_b200 as w4
    from w4a4_int4_quantized_b200 import inputs
    w4.load_library()
    spec = inputs.WORKLOADS["attn_proj"]
    N, K, g, rl = spec.N, spec.K, spec.group, args.bake_lora

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    W = dev(inputs.make_layer(spec)["W"])
    A = dev(inputs.random_bf16((K, rl), seed=11, std=0.05))
    B = dev(inputs.random_bf16((rl, N), seed=12, std=0.05))
    Wb = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
    Wq = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    ws = torch.empty((N,), dtype=torch.float32, device="cuda")
    for i in range(args.warmup):
        w4.w4a4_bake_lora_sr(W, A, B, 1.0, g, i, W_baked=Wb, Wq=Wq, w_scale=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        w4.w4a4_bake_lora_sr(W, A, B, 1.0, g, 1000 + i, W_baked=Wb, Wq=Wq, w_scale=ws)
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) / args.steps * 1e3
    err = w4.w4a4_get_device_error()
    if err:
        raise SystemExit(f"device error word {err:#x}")
    print(json.dumps({
        "metric": f"LoRA bake (rank {rl}) + stochastic-rounding INT4 re-quantization, us per call (N=K=3072)",
        "value": us, "unit": "us", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16 in, fp32 bake, int4 out",
        "data": "synthetic", "config": {"workload": "attn_proj_weights_bake", "N": N, "K": K, "group": g,
                                        "lora_rank": rl},
        "gpu_launches": 2 * args.steps}), flush=True)


def run_block(args):
    """The double-stream block at batch 2 (M = 9216, g = 128): fused QKV
    3072 -> 9216, out-projection 3072 -> 3072, MLP 3072 -> 12288 (GELU fused)
    -> 3072, all W4A4 with rank 64; the W8A8 first and last projections
    (3072 -> 3072) and the timestep MLP layer (256 -> 3072 at M = 2).  Each
    layer runs as its whole-layer call (activation quantization + GEMM);
    per-layer and whole-block device times."""
    import torch
    import w4a4_int4_quantized_b200 as w4
    from w4a4_int4_quantized_b200 import inputs
    w4.load_library()
    names = ["block_first_w8a8", "block_qkv", "block_out", "block_mlp_up", "block_mlp_down", "block_last_w8a8",
             "block_tmlp_w8a8"]

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    layers = []
    for nm in names:
        sp = inputs.WORKLOADS[nm]
        d = inputs.make_layer(sp)
        L = dict(spec=sp, X=dev(d["X"]), bias=dev(d["bias"]) if d["bias"] is not None else None,
                 Y=torch.empty((sp.M, sp.N), dtype=torch.bfloat16, device="cuda"))
        if sp.w8a8:
            L["Wq"], L["ws"] = w4.w8a8_quantize_weights(dev(d["W"]), sp.group)
            L["wsp"] = torch.empty((w4.w8a8_workspace_bytes(sp.M, sp.K),), dtype=torch.uint8, device="cuda")
        else:
            L["Wq"], L["ws"] = w4.w4a4_quantize_weights(dev(d["W"]), sp.group)
            L["L1"], L["L2"] = dev(d["L1"]), dev(d["L2"])
            L["wsp"] = torch.empty((w4.w4a4_workspace_bytes(sp.M, sp.K, sp.rank),), dtype=torch.uint8,
                                   device="cuda")
        layers.append(L)

    def run(L):
        sp = L["spec"]
        if sp.w8a8:
            w4.w8a8_linear(L["X"], L["Wq"], L["ws"], sp.group, L["bias"], Y=L["Y"], workspace=L["wsp"])
        elif sp.name == "block_mlp_up":
            w4.w4a4_linear_gelu(L["X"], L["Wq"], L["ws"], sp.group, L["L1"], L["L2"], L["bias"], Y=L["Y"],
                                workspace=L["wsp"])
        else:
            w4.w4a4_linear(L["X"], L["Wq"], L["ws"], sp.group, L["L1"], L["L2"], L["bias"], Y=L["Y"],
                           workspace=L["wsp"])

    def timed(fn, n):
        # n calls captured in a CUDA graph and replayed (host time per call
        # would otherwise pace the small layers)
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            for _ in range(n):
                fn()
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        torch.cuda.synchronize()
        del graph
        return e0.elapsed_time(e1) / n * 1e3

    per = {L["spec"].name: timed(lambda L=L: run(L), args.steps) for L in layers}

    def block():
        for L in layers:
            run(L)

    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    t0 = time.perf_counter()
    us = timed(block, args.steps)
    clocks.mark(t0, time.perf_counter())
    clk = clocks.stop()
    ops = sum(2.0 * L["spec"].M * L["spec"].N * L["spec"].K for L in layers)
    err = w4.w4a4_get_device_error()
    if err:
        raise SystemExit(f"device error word {err:#x}")
    print(json.dumps({
        "metric": "Flux-like double-stream block at batch 2 (M=9216): us per block of linear layers",
        "value": us, "unit": "us", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": us / 1e3,
        "tops": ops / (us * 1e-6) / 1e12, "per_layer_us": per,
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "int4 / int8 codes (int8 MMA, int32 acc), bf16 in/out", "data": "synthetic",
        "config": {"workload": "block_batch2", "M": 9216, "group": 128, "rank": 64},
        "gpu_launches": sum(2 if L["spec"].w8a8 else 3 for L in layers) * args.steps, "clocks": clk}), flush=True)


def run_sweep(args):
    """Shape sweep (one GPU): M in {256, 1024, 4608, 9216, 16384} x (K, N) in
    {(3072, 3072), (3072, 9216), (3072, 12288), (12288, 3072)} x rank in
    {0, 16, 64, 128} for W4A4 (group 128), plus the W4A8 layer at every
    (M, K, N), and the tiny single layer (M=64, K=N=256, group 64, rank 16).
    Inputs: X ~ N(0,1) with 1% of channels x100, W ~ N(0, 0.02), L1, L2 ~
    N(0, 0.01), bias ~ N(0, 0.01), drawn on the device from fixed seeds.  Each
    point: the whole-layer call (w4a4_linear / w4a8_linear), L2 flushed before
    every timed call (a 256 MB write outside the events), CUDA events around
    the call, median over --steps calls.  One JSON line per point."""
    import torch
    import w4a4_int4_quantized_b200 as w4
    w4.load_library()
    torch.cuda.set_device(0)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    pk = _peaks()
    i8 = 2.0 * pk["bf16"]
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.3)
    t0 = time.perf_counter()

    def draw(shape, seed, std):
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    def acts(M, K, seed):
        X = torch.randn((M, K), generator=torch.Generator(device="cuda").manual_seed(seed), device="cuda")
        ch = torch.randperm(K, generator=torch.Generator(device="cuda").manual_seed(seed + 1), device="cuda")
        X[:, ch[: max(1, round(0.01 * K))]] *= 100.0
        return X.to(torch.bfloat16)

    def graph_of(fn, with_flush):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            if with_flush:
                flush.fill_(1)
            if fn is not None:
                fn(torch.cuda.current_stream())
        return g

    def replay_us(g, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g.replay()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(n):
            g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) * 1e3 / n

    g_flush = graph_of(None, True)

    def timed(fn):
        # the layer call and a 256 MB L2 flush replayed from one CUDA graph,
        # back to back (no host time between calls), minus the flush alone
        for _ in range(args.warmup):
            fn(stream)
        torch.cuda.synchronize()
        g = graph_of(fn, True)
        n = max(args.steps, 5)
        us = min(replay_us(g, n) - replay_us(g_flush, n) for _ in range(3))
        del g
        return us

    def emit(name, M, K, N, g, r, variant, us, code_bytes):
        ops = 2.0 * M * N * K
        lr = 2.0 * M * r * (K + N)
        wbytes = N * K // 2 if variant != "w8a8" else N * K
        bytes_ = M * K * 2 + M * N * 2 + wbytes + (M * r * 2 * 2 + (K + N) * r * 2 if r else 0) + code_bytes
        roof_us = max((ops / (4500e12) + lr / (2250e12)) * 1e6, bytes_ / (pk["hbm_gbs"] * 1e9) * 1e6)
        print(json.dumps({"sweep": name, "variant": variant, "M": M, "K": K, "N": N, "group": g, "rank": r,
                          "us": us, "tops": ops / (us * 1e-6) / 1e12,
                          "frac_of_int8_nominal": ops / (us * 1e-6) / 1e12 / INT8_NOMINAL_TOPS,
                          "frac_of_int8_measured": ops / (us * 1e-6) / 1e12 / i8,
                          "roofline_us": roof_us, "frac_of_roofline": roof_us / us,
                          "l2": "flushed before every call (the flush time is subtracted)"}), flush=True)

    # the tiny single layer
    X = acts(64, 256, 0)
    Wq, ws = w4.w4a4_quantize_weights(draw((256, 256), 1, 0.02), 64)
    L1, L2 = draw((256, 16), 2, 0.01), draw((16, 256), 3, 0.01)
    ws_buf = torch.empty((w4.w4a4_workspace_bytes(64, 256, 16),), dtype=torch.uint8, device="cuda")
    Y = torch.empty((64, 256), dtype=torch.bfloat16, device="cuda")
    us = timed(lambda st: w4.w4a4_linear(X, Wq, ws, 64, L1, L2, None, Y=Y, workspace=ws_buf, stream=st))
    emit("tiny", 64, 256, 256, 64, 16, "w4a4", us, 64 * 128)

    Ms = [256, 1024, 4608, 9216, 16384]
    KN = [(3072, 3072), (3072, 9216), (3072, 12288), (12288, 3072)]
    ranks = [0, 16, 64, 128]
    for ki, (K, N) in enumerate(KN):
        seed = 1000 + 10 * ki
        W = draw((N, K), seed, 0.02)
        Wq, ws = w4.w4a4_quantize_weights(W, 128)
        Wq8, ws8, wz8 = w4.w4a8_quantize_weights(W, 128)
        b = draw((N,), seed + 1, 0.01)
        L1f, L2f = draw((K, 128), seed + 2, 0.01), draw((128, N), seed + 3, 0.01)
        del W
        for M in Ms:
            X = acts(M, K, seed + 5 + M)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            for r in ranks:
                L1 = L1f[:, :r].contiguous() if r else None
                L2 = L2f[:r].contiguous() if r else None
                wsb = torch.empty((w4.w4a4_workspace_bytes(M, K, r),), dtype=torch.uint8, device="cuda")
                us = timed(lambda st: w4.w4a4_linear(X, Wq, ws, 128, L1, L2, b, Y=Y, workspace=wsb, stream=st))
                emit("c5", M, K, N, 128, r, "w4a4", us, M * K // 2)
                del wsb
            wsb = torch.empty((w4.w4a8_workspace_bytes(M, K),), dtype=torch.uint8, device="cuda")
            us = timed(lambda st: w4.w4a8_linear(X, Wq8, ws8, wz8, 128, b, Y=Y, workspace=wsb, stream=st))
            emit("c5", M, K, N, 128, 0, "w4a8", us, M * K)
            del X, Y, wsb
            torch.cuda.empty_cache()
    clocks.mark(t0, time.perf_counter())
    clk = clocks.stop()
    err = w4.w4a4_get_device_error()
    if err:
        raise SystemExit(f"device error word {err:#x}")
    print(json.dumps({"sweep": "done", "clocks": clk, "peaks": pk}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="attn_proj")
    ap.add_argument("--sets", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--soak-ms", type=float, default=400.0,
                    help="run blocks of --steps steps for this long before the timed region (clock record)")
    ap.add_argument("--sweep", action="store_true",
                    help="shape sweep: M x (K, N) x rank for W4A4 plus the W4A8 points, one JSON line each")
    ap.add_argument("--block", action="store_true",
                    help="time the linear layers of the double-stream block at batch 2 (M=9216)")
    ap.add_argument("--bake-lora", type=int, default=0,
                    help="time baking a LoRA of this rank into the weights with stochastic re-quantization")
    ap.add_argument("--mlp", action="store_true",
                    help="time the fused MLP pair (up with GELU in its epilogue, then down) instead")
    ap.add_argument("--lora", type=int, default=0,
                    help="rank of a runtime LoRA merged beside the layer's low-rank branch (w4a4)")
    ap.add_argument("--variant", choices=["w4a4", "w4a8"], default="w4a4",
                    help="w4a8: rotated int8 activations x zero-pointed 4-bit weights")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    from w4a4_int4_quantized_b200 import inputs
    if args.sweep:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the sweep is measured by the GPU arm only"}))
            return
        run_sweep(args)
        return
    if args.block:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the block is measured by the GPU arm only"}))
            return
        run_block(args)
        return
    if args.bake_lora:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the bake is measured by the GPU arm only"}))
            return
        run_bake(args)
        return
    if args.mlp:
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the MLP chain is measured by the GPU arm only"}))
            return
        run_mlp(args)
        return
    spec = inputs.WORKLOADS[args.workload]
    w4a8 = args.variant == "w4a8"
    if w4a8 and (spec.rank or args.lora):
        raise SystemExit("the W4A8 path has no low-rank branch: pick a workload with rank 0 and no --lora")
    if args.impl == "reference":
        run_reference(args, spec)
        return

    import torch
    import torch.distributed as dist
    import w4a4_int4_quantized_b200 as w4

    rank, world, local = _dist_init(args.gpus)
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    w4.load_library()
    g, M, K, N, r = spec.group, spec.M, spec.K, spec.N, spec.rank + args.lora

    def dev(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()

    sets = []
    for i in range(args.sets):
        d = inputs.make_layer(spec, seed_offset=1000 * rank + i)
        X = dev(d["X"])
        if w4a8:
            Wq, ws, wz = w4.w4a8_quantize_weights(dev(d["W"]), g)
        else:
            (Wq, ws), wz = w4.w4a4_quantize_weights(dev(d["W"]), g), None
        L1 = dev(d["L1"]) if spec.rank else None
        L2 = dev(d["L2"]) if spec.rank else None
        if args.lora:
            # runtime LoRA (A, B ~ N(0, 0.01), scale 1) merged into one branch
            A = dev(inputs.random_bf16((K, args.lora), seed=7000 + i, std=0.01))
            B = dev(inputs.random_bf16((args.lora, N), seed=8000 + i, std=0.01))
            L1, L2 = w4.w4a4_lora_merge(L1, L2, A, B, 1.0)
        s = dict(X=X, Wq=Wq, ws=ws, wz=wz, bias=dev(d["bias"]) if d["bias"] is not None else None,
                 L1=L1, L2=L2,
                 Xq=(torch.empty((M, K), dtype=torch.int8, device="cuda") if w4a8 else
                     torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")),
                 xs=torch.empty((M,), dtype=torch.float32, device="cuda"),
                 T=torch.empty((M, r), dtype=torch.bfloat16, device="cuda") if r else None,
                 Y=torch.empty((M, N), dtype=torch.bfloat16, device="cuda"))
        s["work"] = torch.empty((w4.w4a8_workspace_bytes(M, K) if w4a8 else w4.w4a4_workspace_bytes(M, K, r),),
                                dtype=torch.uint8, device="cuda")
        sets.append(s)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def k1(s, st=None):
        st = stream if st is None else st
        if w4a8:
            w4.w8a8_rotate_quantize_act(s["X"], g, Xq=s["Xq"], x_scale=s["xs"], stream=st)
        else:
            w4.w4a4_rotate_quantize_act(s["X"], g, s["L1"], Xq=s["Xq"], x_scale=s["xs"], T=s["T"], stream=st)

    def k2(s, st=None):
        st = stream if st is None else st
        if w4a8:
            w4.w4a8_gemm(s["Xq"], s["xs"], s["Wq"], s["ws"], s["wz"], g, s["bias"], Y=s["Y"], stream=st)
        else:
            w4.w4a4_gemm(s["Xq"], s["xs"], s["Wq"], s["ws"], g, s["T"], s["L2"], s["bias"], Y=s["Y"],
                         stream=st)

    def step(s, st=None):
        # one whole layer through the public call (its kernels: rotate +
        # quantize, the low-rank down-projection when r > 0, the GEMM)
        st = stream if st is None else st
        if w4a8:
            w4.w4a8_linear(s["X"], s["Wq"], s["ws"], s["wz"], g, s["bias"], Y=s["Y"], workspace=s["work"],
                           stream=st)
        else:
            w4.w4a4_linear(s["X"], s["Wq"], s["ws"], g, s["L1"], s["L2"], s["bias"], Y=s["Y"], workspace=s["work"],
                           stream=st)

    for i in range(args.warmup):
        step(sets[i % len(sets)])
    torch.cuda.synchronize()
    # The K steps of the timed region are captured once as a CUDA graph (the
    # way a server runs a fixed-shape layer: one replay launches every kernel
    # of the K layers, with the same programmatic-launch overlap between
    # them), so that the host's per-call cost is not timed as GPU work.  The
    # same K calls launched one by one from the host are timed after it
    # (`us_per_layer_direct`).
    steps_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(steps_graph, capture_error_mode="thread_local"):
        for i in range(args.steps):
            step(sets[i % len(sets)], torch.cuda.current_stream())

    def replay_steps():
        with torch.cuda.stream(stream):
            steps_graph.replay()

    replay_steps()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    # clock soak: blocks of K steps back to back for --soak-ms (untimed for
    # `value`; each block timed on its own for the `sustained` figure), so the
    # clock record sampled across soak + timed region covers the clock the
    # timed steps ran at, however short they are
    e_blk = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    soak_ms, soak_blocks = [], 0
    wall0 = time.perf_counter()
    while args.soak_ms > 0 and (time.perf_counter() - wall0) * 1e3 < args.soak_ms:
        e_blk[0].record(stream)
        replay_steps()
        e_blk[1].record(stream)
        e_blk[1].synchronize()
        soak_ms.append(e_blk[0].elapsed_time(e_blk[1]) / args.steps)
        soak_blocks += 1
    if world > 1:
        # every rank takes the same collective steps: agree on the block count
        nb = torch.tensor([soak_blocks], device="cuda")
        dist.all_reduce(nb, op=dist.ReduceOp.MAX)
        for _ in range(int(nb.item()) - soak_blocks):
            replay_steps()
        torch.cuda.synchronize()
        dist.barrier()
    # timed region: K whole layers back to back (no events between kernels,
    # so each launch may overlap the previous kernel's tail)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_timed = time.perf_counter()
    e_start.record(stream)
    replay_steps()
    e_end.record(stream)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t_timed
    total_ms = e_start.elapsed_time(e_end)
    if world > 1:
        dist.barrier()
    # the same K layers launched call by call from the host, right after (the
    # clock still at its loaded value)
    e_start.record(stream)
    t_host = time.perf_counter()
    for i in range(args.steps):
        step(sets[i % len(sets)])
    host_us = (time.perf_counter() - t_host) / args.steps * 1e6   # host time to issue one call
    e_end.record(stream)
    torch.cuda.synchronize()
    direct_ms = e_start.elapsed_time(e_end)
    clocks.mark(wall0, t_timed + wall)
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    del steps_graph

    # per-kernel durations for the roofline: each kernel alone, back to back,
    # on the same rotating sets, replayed from a CUDA graph so that the host's
    # per-call cost (Python and argument checks, ~10 us) does not set the
    # pace of the short kernels (CUDA events on the replaying stream)
    def timed(fn, n):
        for i in range(3):
            fn(sets[i % len(sets)])
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, capture_error_mode="thread_local"):
            for i in range(n):
                fn(sets[i % len(sets)], torch.cuda.current_stream())
        graph.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        with torch.cuda.stream(stream):
            graph.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del graph
        return a.elapsed_time(b) / n

    n_split = min(args.steps, 200)
    k1_ms = timed(k1, n_split)
    k2_ms = timed(k2, n_split)
    err = w4.w4a4_get_device_error()
    if err:
        raise SystemExit(f"device error word {err:#x}")
    from w4a4_int4_quantized_b200.shard import max_over_ranks
    total_ms = max_over_ranks(total_ms, device="cuda")
    direct_ms = max_over_ranks(direct_ms, device="cuda")
    ops = 2.0 * M * N * K
    value = ops * args.steps * world / (total_ms * 1e-3) / 1e12

    # end to end through the public call: pinned host X in, host Y out.
    # Steps are pipelined the way a server would run them: two device buffer
    # sets, the host-to-device copy of step i+1 and the device-to-host copy of
    # step i-1 on their own streams beside the layer of step i (PCIe is full
    # duplex), ordered by events; every step still makes its own two copies
    # inside the timed region.
    e2e = None
    if args.e2e_steps > 0:
        s = sets[0]
        hx = [torch.empty((M, K), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        for h in hx:
            h.copy_(s["X"].cpu())
        hy = [torch.empty((M, N), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
        dX = [torch.empty_like(s["X"]) for _ in range(2)]
        dY = [torch.empty_like(s["Y"]) for _ in range(2)]
        ws_buf = [torch.empty((w4.w4a8_workspace_bytes(M, K) if w4a8 else w4.w4a4_workspace_bytes(M, K, r),),
                              dtype=torch.uint8, device="cuda") for _ in range(2)]
        s_h2d, s_cmp, s_d2h = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

        def linear(b, st):
            if w4a8:
                w4.w4a8_linear(dX[b], s["Wq"], s["ws"], s["wz"], g, s["bias"], Y=dY[b], workspace=ws_buf[b],
                               stream=st)
            else:
                w4.w4a4_linear(dX[b], s["Wq"], s["ws"], g, s["L1"], s["L2"], s["bias"], Y=dY[b],
                               workspace=ws_buf[b], stream=st)

        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_cmp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def pipelined(n):
            # buffer set b = i % 2: the copy into dX[b] waits for the layer
            # two steps back (the last reader of dX[b]), the layer for the
            # copy-out two steps back (the last reader of dY[b])
            for i in range(n):
                b = i & 1
                if i >= 2:
                    s_h2d.wait_event(ev_cmp[b])
                with torch.cuda.stream(s_h2d):
                    dX[b].copy_(hx[b], non_blocking=True)
                ev_in[b].record(s_h2d)
                s_cmp.wait_event(ev_in[b])
                if i >= 2:
                    s_cmp.wait_event(ev_out[b])
                linear(b, s_cmp)
                ev_cmp[b].record(s_cmp)
                s_d2h.wait_event(ev_cmp[b])
                with torch.cuda.stream(s_d2h):
                    hy[b].copy_(dY[b], non_blocking=True)
                ev_out[b].record(s_d2h)
            return ev_out[(n - 1) & 1]

        pipelined(3)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_h2d)
        s_cmp.wait_stream(s_h2d)
        s_d2h.wait_stream(s_h2d)
        last = pipelined(args.e2e_steps)
        stream.wait_event(last)
        stream.wait_stream(s_cmp)
        stream.wait_stream(s_h2d)
        e1.record(stream)
        torch.cuda.synchronize()
        te = max_over_ranks(e0.elapsed_time(e1), device="cuda")
        # one step at a time, with events between its three parts (for the split)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        parts = [0.0, 0.0, 0.0]
        for _ in range(args.e2e_steps):
            ev[0].record(stream)
            dX[0].copy_(hx[0], non_blocking=True)
            ev[1].record(stream)
            linear(0, stream)
            ev[2].record(stream)
            hy[0].copy_(dY[0], non_blocking=True)
            ev[3].record(stream)
            torch.cuda.synchronize()
            for j in range(3):
                parts[j] += ev[j].elapsed_time(ev[j + 1])
        e2e = {"value": ops * args.e2e_steps * world / (te * 1e-3) / 1e12, "unit": "TOPS",
               "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
               "us_per_step": te / args.e2e_steps * 1e3,
               "split_us": {"h2d": parts[0] / args.e2e_steps * 1e3, "layer": parts[1] / args.e2e_steps * 1e3,
                            "d2h": parts[2] / args.e2e_steps * 1e3,
                            "note": "one step alone: pinned host copies over PCIe around one w4a4_linear call; "
                                    "the timed steps overlap step i's layer with the copies of its neighbours"}}

    if rank == 0:
        pk = _peaks()
        k1 = k1_ms
        k2 = k2_ms
        k2_tops = ops / (k2 * 1e-3) / 1e12
        # the GEMM is timed alone in a short back-to-back loop at full clock:
        # the burst bf16 figure x the nominal int8 : bf16 ratio of 2
        int8_peak = 2.0 * pk["bf16"]
        k1_bytes = M * K * 2 + (M * K if w4a8 else M * K // 2) + M * 4
        adj = clock_adjusted_peak_tops(clk.get("sm_mhz"))
        line = {
            "metric": _metric_name(args.variant, spec),
            "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "us_per_layer": total_ms / args.steps * 1e3,
            "us_per_layer_direct": direct_ms / args.steps * 1e3, "host_us_per_call": host_us,
            "frac_of_int8_nominal_peak": value / INT8_NOMINAL_TOPS,
            "layer_frac": {"of_int8_nominal": value / INT8_NOMINAL_TOPS,
                           "of_int8_measured": value / world / (2.0 * pk["bf16"]),
                           "of_int8_clock_adjusted": (value / world / adj) if adj else None,
                           "clock_adjusted_peak_tops": adj,
                           "note": "whole layer (K1 + K2) per GPU; clock-adjusted = 8192 int8 MAC/clk/SM x 2 x "
                                   "148 SMs x median sampled SM clock"},
            "sustained": {"us_per_layer_median": statistics.median(soak_ms) * 1e3 if soak_ms else None,
                          "blocks": len(soak_ms), "steps_per_block": args.steps,
                          "note": "blocks of K steps run back to back before the timed region (clock soak)"},
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("int8 activations x 4-bit zero-pointed weights" if w4a8 else "int4 codes")
                     + " (int8 MMA, int32 acc), bf16 in/out", "data": "synthetic",
            "config": {"workload": spec.name, "variant": args.variant, "M": M, "K": K, "N": N, "group": g, "rank": r,
                       "lora_rank": args.lora,
                       "bias": spec.bias, "parallelism": f"replicas x{world} (token shards, no exchange)",
                       "l2": f"{args.sets} rotating input sets (> L2)",
                       "launch": f"the K steps captured once as a CUDA graph of {'w4a8' if w4a8 else 'w4a4'}_linear "
                                 "calls, replayed in the timed region (us_per_layer_direct: the same calls launched "
                                 "one by one)",
                       "clock_soak_ms": args.soak_ms},
            "split_us": {"rotate_quantize": k1 * 1e3, "gemm": k2 * 1e3,
                         "note": "each kernel timed alone, back to back, replayed from a CUDA graph"},
            "roofline": {"bound": "tensor", "achieved": k2_tops, "peak": int8_peak, "unit": "TOPS",
                         "frac": k2_tops / int8_peak,
                         "frac_clock_adjusted": (k2_tops / adj) if adj else None,
                         "traffic": None if r else _traffic("gemm_w4a8" if w4a8 else "gemm", spec.name),
                         "peak_note": f"int8 = 2 x {pk['source']} burst bf16 {pk['bf16']} TFLOP/s (kernel timed "
                                      f"alone); {2.0 * pk['bf16_sustained']:.0f} with the sustained figure"},
            "roofline_k1": {"bound": "hbm", "achieved": k1_bytes / (k1 * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                            "unit": "GB/s", "frac": k1_bytes / (k1 * 1e-3) / 1e9 / pk["hbm_gbs"],
                            "traffic": None if (w4a8 or r) else _traffic("rotate_quantize", spec.name)},
            "gpu_launches": 2 * args.steps + (args.steps if r else 0),
            "clocks": clk, "wall_s": wall, "e2e": e2e,
        }
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(spec, variant=args.variant)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
