#!/usr/bin/env python3
"""BitLinear benchmark on B200: one JSON line per run (rank 0).

Headline (the default): the 70B-class prefill BitLinear, M = 4096 tokens of bf16
activations against a 28672 x 8192 ternary weight matrix (K = 8192 -> N = 28672). A step is
one BitLinear forward of the batch: per-token int8 quantization of the activations, the
exact int32 contraction on the tcgen05 int8 tensor cores and the rescale to bf16. The
weights are quantized once before the timed region (absmean gamma, ternary codes, 2-bit
packing), as a deployed layer holds them; the weight quantization is timed on its own and
reported in the same line, over every 70B-shaped layer matrix, together with the decode
shapes (70B up/down, 700M up) and, where built, the 3B 26-layer FFN chain.

The timed loops replay CUDA graphs captured from the library calls, so host launch
overhead is not part of the kernel numbers; `e2e` times the plain library calls with host
buffers (host->device copy of the batch, forward, device->host copy of the output).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--M M] [--no-others] [--no-cpu-baseline] [--no-e2e]

Multi-GPU (torchrun): every rank runs the same per-GPU workload on its own weights and
batch (weak scaling, no data-path collective); timing is the max over ranks.
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
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ternary_weight_linear_03_b200 import dist as bldist  # noqa: E402
from ternary_weight_linear_03_b200 import synthetic as syn  # noqa: E402

METRIC = "BitLinear tokens/s; decode HBM GB/s and prefill INT8 TOPS as % of roofline"
L2_BYTES = 126 * 1024 * 1024
HEADLINE = "70b_prefill_4096x8192x28672"
EPS = 1e-5


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=HEADLINE)
    p.add_argument("--M", type=int, default=None, help="tokens (default: the workload's largest)")
    p.add_argument("--no-others", action="store_true", help="skip the secondary figures")
    p.add_argument("--figure", default="headline",
                   choices=["headline", "decode", "decode_base3", "weight_quant", "sweep",
                            "backward"],
                   help="run one secondary figure alone and print it (for profiling)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    a = p.parse_args()
    if a.M is None:
        a.M = max(syn.WORKLOADS[a.workload]["Ms"])
    return a


KERNEL_SOURCES = {"weight_quant_kernel": "weight_quant.cuh",
                  "gemm_prefill_kernel": "gemm_prefill.cuh",
                  "gemm_skinny_kernel": "gemm_skinny.cuh", "gemv_kernel": "gemv.cuh"}


def ncu_traffic(kernel: str, workload: str, M: int):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when the
    capture was of another workload or the kernel source changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "ternary_weight_linear_03_b200", "csrc", KERNEL_SOURCES[kernel])
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
        with open(src, "rb") as f:
            sha = hashlib.sha1(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("workload") != workload or rec.get("M") != M or rec.get("source_sha1") != sha:
        return None
    return rec["dram_bytes_per_launch"]


def peaks():
    """(HBM GB/s, bf16 burst TFLOP/s, bf16 sustained TFLOP/s, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]),
                float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


# ----------------------------------------------------------------------------- clocks


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nvml = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nvml.nvmlDeviceGetClockInfo(self._h, self._nvml.NVML_CLOCK_SM))
                mask = self._nvml.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nvml is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nvml is not None:
            self._t.join()

    def result(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- oracle arm


class OracleSample:
    """A bounded sample of one forward step for the oracle (plain single-threaded C++ on
    the host): the first T tokens against the first R weight rows. The weights are
    quantized once beforehand (gamma over those rows), as on the GPU side. The work of a
    step is linear in tokens x rows (quantizing T activation rows is a small part), so a
    full step takes (M * N) / (T * R) times as long and tokens/s = T * R / (N * step time)."""

    def __init__(self, name: str, M: int):
        from oracle import oracle as orc
        self.orc = orc
        wl = syn.WORKLOADS[name]
        self.N, self.K, self.M = wl["N"], wl["K"], M
        self.T = min(M, 16)
        self.R = min(self.N, 256 if M > 64 else 512)
        W = syn.weights(self.R, self.K, wl["sigma"], seed=syn.w_seed(name))
        x = syn.activations(self.T, self.K, seed=syn.x_seed(name, M), dtype=wl["x_dtype"],
                            outlier_frac=wl["outlier_frac"])
        self.xin = syn.bf16_bits(x) if x.dtype == torch.bfloat16 else x.numpy()
        self.packed, self.gamma = orc.quantize_weights(W.numpy(), EPS)
        self.name = name

    def step(self):
        self.orc.forward(self.xin, self.packed, self.gamma, out="bf16")

    def tokens_per_s(self, seconds_per_step: float) -> float:
        return self.T * self.R / (self.N * seconds_per_step)

    def describe(self, steps: int, elapsed: float) -> str:
        return (f"{steps} steps of tokens 0..{self.T - 1} x weight rows 0..{self.R - 1} of the "
                f"{self.name} forward (M={self.M}, N={self.N}, K={self.K}; act quant, int32 "
                f"contraction, rescale to bf16), single-threaded C++ oracle, {elapsed:.1f} s; "
                f"scaled by (M*N)/(T*R) = {self.M * self.N / (self.T * self.R):.0f} "
                f"(work is linear in tokens x rows)")


def cpu_baseline(name: str, M: int, budget_s: float = 12.0):
    """The oracle, as it stands, on this host for about budget_s seconds."""
    s = OracleSample(name, M)
    steps, t0 = 0, time.perf_counter()
    while True:
        s.step()
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": s.tokens_per_s(el / steps), "unit": "tokens/s", "cores": 1,
            "kind": "oracle", "sample": s.describe(steps, el)}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    s = OracleSample(args.workload, args.M)
    for _ in range(args.warmup):
        s.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.step()
    el = time.perf_counter() - t0
    value = s.tokens_per_s(el / args.steps)
    wl = syn.WORKLOADS[args.workload]
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8xternary->i32 (bf16 in/out)", "data": "synthetic",
        "config": config_of(args.workload, args.M, wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": s.describe(args.steps, el)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def config_of(name: str, M: int, wl: dict, world: int) -> dict:
    return {"workload": name, "M": M, "N": wl["N"], "K": wl["K"], "w_dtype": "fp32",
            "x_dtype": str(wl["x_dtype"]).replace("torch.", ""), "out": "bf16",
            "weights": "quantized once before the timed region (2-bit packed, resident)",
            "parallelism": f"replicas x{world}"}


# ----------------------------------------------------------------------------- GPU helpers


def time_back_to_back(calls, reps: int = 5):
    """Mean device time (ms) per call of a list of library calls run back to back: one CUDA
    graph holding them all, replayed `reps` times between two events (the steady state of
    a stream of such calls, inter-kernel gaps included)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for c in calls:
            c()
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(reps):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    del g
    return s.elapsed_time(e) / (reps * len(calls))


def forward_launches(bl, M: int, N: int, K: int) -> int:
    """Kernels one bitlinear_forward launches (the GEMV alone, or activation quantization
    followed by a tensor-core kernel), from the library's own plan."""
    path, _ = bl.debug_plan(M, N, K, sms=torch.cuda.get_device_properties(0).multi_processor_count)
    return 1 if path == "gemv" else 2


def packed_copies(bl, name: str, device, copies: int, seed_offset: int = 0):
    """`copies` device copies of one quantized weight matrix of the workload (distinct
    addresses, so rotating through them reads every step's weights from HBM)."""
    wl = syn.WORKLOADS[name]
    W = syn.weights(wl["N"], wl["K"], wl["sigma"], seed=syn.w_seed(name) + seed_offset,
                    device=device)
    packed, gamma = bl.quantize_weights(W, EPS)
    del W
    out = [(packed, gamma)] + [(packed.clone(), gamma.clone()) for _ in range(copies - 1)]
    torch.cuda.synchronize()
    return out


def act_copies(name: str, M: int, device, copies: int, seed_offset: int = 0):
    wl = syn.WORKLOADS[name]
    return [syn.activations(M, wl["K"], seed=syn.x_seed(name, M) + 97 * i + seed_offset,
                            dtype=wl["x_dtype"], outlier_frac=wl["outlier_frac"], device=device)
            for i in range(copies)]


def decode_figure(bl, name: str, M: int, device, hbm_peak: float, i8_peak: float):
    """One forward shape timed alone: mean device time per launch over rotated copies of the
    weights (more than twice L2 in total), GB/s of algorithmic bytes, int8 TOPS, fractions."""
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    w_bytes = N * K // 4
    copies = max(2, math.ceil(2 * L2_BYTES / w_bytes))
    ws = packed_copies(bl, name, device, copies)
    xs = act_copies(name, M, device, min(copies, 8))
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    work = bl.workspace(M, N, K, device)
    calls = [(lambda i=i: bl.forward(xs[i % len(xs)], ws[i][0], ws[i][1], y=y, ws=work))
             for i in range(copies)]
    for c in calls[:2]:
        c()
    torch.cuda.synchronize()
    ms = time_back_to_back(calls)
    alg_bytes = w_bytes + M * K * 2 + M * N * 2
    ops = 2.0 * M * N * K
    gbs = alg_bytes / (ms * 1e-3) / 1e9
    tops = ops / (ms * 1e-3) / 1e12
    bound = "hbm" if alg_bytes / (hbm_peak * 1e9) >= ops / (i8_peak * 1e12) else "tensor"
    path, splits = bl.debug_plan(M, N, K)
    return {"workload": name, "M": M, "kernel": path, "k_splits": splits, "ms": ms,
            "GBps": gbs, "frac_hbm": gbs / hbm_peak, "TOPS": tops, "frac_i8": tops / i8_peak,
            "bound": bound, "tokens_per_s": M / (ms * 1e-3), "weight_copies": copies}


def sweep_3b_figures(bl, device, hbm_peak: float, Ms=(1, 16, 64), blocks: int = 26):
    """The 3B-class feed-forward sweep: 26 blocks of gate and up (3200 -> 8640, one shared
    input) and down (8640 -> 3200, reading up; the elementwise activation between them is
    not part of BitLinear), 78 matrices and 539 MB of packed weights, as one
    bitlinear_chain_forward captured in a CUDA graph; next to it the same 78 forwards as
    separate bitlinear_forward calls (each quantizing its own input) in one graph."""
    d, h = 3200, 8640
    layers, src = [], -1
    for b in range(blocks):
        for i, (N, K) in enumerate([(h, d), (h, d), (d, h)]):
            W = syn.weights(N, K, 0.02, seed=9000 + 3 * b + i, device=device)
            packed, gamma = bl.quantize_weights(W, EPS)
            del W
            layers.append([packed, gamma, src if i < 2 else len(layers) - 1])
        src = len(layers) - 1
    torch.cuda.synchronize()
    w_bytes = sum(ly[0].numel() for ly in layers)
    rows = []
    for M in Ms:
        gate = torch.empty((M, h), dtype=torch.bfloat16, device=device)
        chain = [(p_, g_, s_, gate) if i % 3 == 0 else (p_, g_, s_)
                 for i, (p_, g_, s_) in enumerate(layers)]
        x = syn.activations(M, d, seed=77 + M, device=device)
        y = torch.empty((M, d), dtype=torch.bfloat16, device=device)
        ws = bl.chain_workspace(M, chain, device)
        bl.chain_forward(x, chain, y=y, ws=ws)
        torch.cuda.synchronize()
        ms_chain = time_back_to_back([lambda: bl.chain_forward(x, chain, y=y, ws=ws)] * 4)
        # unchained: separate forwards, each quantizing its input itself
        bufs = {-1: x}
        outs = [torch.empty((M, ly[0].shape[0]), dtype=torch.bfloat16, device=device)
                for ly in layers]
        fws = torch.empty(max(bl.workspace_size(M, h, d), bl.workspace_size(M, d, h)),
                          dtype=torch.uint8, device=device)

        def separate():
            for i, (p_, g_, s_) in enumerate(layers):
                bl.forward(bufs[s_] if s_ < 0 else outs[s_], p_, g_, y=outs[i], ws=fws)

        separate()
        torch.cuda.synchronize()
        ms_sep = time_back_to_back([separate] * 2)
        gbs = w_bytes / (ms_chain * 1e-3) / 1e9
        rows.append({"M": M, "ms_per_sweep": ms_chain, "tokens_per_s": M / (ms_chain * 1e-3),
                     "GBps": gbs, "frac_hbm": gbs / hbm_peak,
                     "ms_per_sweep_separate_forwards": ms_sep,
                     "ideal_ms_at_peak": w_bytes / (hbm_peak * 1e9) * 1e3})
        del ws, bufs, outs
    return {"matrices": len(layers), "packed_MB": w_bytes / 1e6, "rows": rows,
            "launches_per_sweep": {"chain": "1 memset + per matrix 1 kernel (GEMV) or "
                                            "act quant once per input + 1 tensor-core kernel"}}


def decode3_figure(bl, name: str, M: int, device, hbm_peak: float):
    """bitlinear_forward_base3 (5 trits per byte) on one decode shape, timed like
    decode_figure over rotated copies of the base-3 weights."""
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    w3_bytes = N * bl.base3_row_bytes(K)
    copies = max(2, math.ceil(2 * L2_BYTES / w3_bytes))
    packed, gamma = packed_copies(bl, name, device, 1)[0]
    p3 = bl.pack_base3(packed)
    ws = [p3] + [p3.clone() for _ in range(copies - 1)]
    xs = act_copies(name, M, device, min(copies, 8))
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    calls = [(lambda i=i: bl.forward_base3(xs[i % len(xs)], ws[i], gamma, y=y))
             for i in range(copies)]
    calls[0]()
    torch.cuda.synchronize()
    ms = time_back_to_back(calls)
    alg = w3_bytes + M * K * 2 + M * N * 2
    gbs = alg / (ms * 1e-3) / 1e9
    return {"workload": name, "M": M, "kernel": "gemv3 (base-3)", "ms": ms, "GBps": gbs,
            "frac_hbm": gbs / hbm_peak, "weight_bytes": w3_bytes,
            "weight_bytes_2bit": N * K // 4, "weight_copies": copies}


def backward_figure(bl, device, bf16_peak: float, M: int = 4096, name: str = "700m_up_1536x4096"):
    """The straight-through backward of one BitLinear layer for a training batch of M tokens
    (bf16 upstream gradient): grad_x (gamma G C) and grad_w (G^T X~) on the tcgen05 bf16
    tensor cores, timed back to back; 2 M N K flops each."""
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    packed, gamma = packed_copies(bl, name, device, 1)[0]
    packedT = bl.pack_transpose(packed)
    x = syn.activations(M, K, seed=11, dtype=torch.bfloat16, device=device)
    G = (syn.activations(M, N, seed=12, dtype=torch.float32, device=device) * 0.01).bfloat16()
    n = bl.load_library().bitlinear_backward_workspace_size(M, N, K)
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    fx = lambda: bl.backward(x, G, packedT, gamma, need_w=False, ws=ws)  # noqa: E731
    fw = lambda: bl.backward(x, G, packedT, gamma, need_x=False, ws=ws)  # noqa: E731
    fx(); fw()
    torch.cuda.synchronize()
    flops = 2.0 * M * N * K
    ms_x = time_back_to_back([fx] * 4)
    ms_w = time_back_to_back([fw] * 4)
    tx = flops / (ms_x * 1e-3) / 1e12
    tw = flops / (ms_w * 1e-3) / 1e12
    return {"workload": name, "M": M, "grad_x_ms": ms_x, "grad_x_TFLOPs": tx,
            "grad_x_frac_bf16": tx / bf16_peak, "grad_w_ms": ms_w, "grad_w_TFLOPs": tw,
            "grad_w_frac_bf16": tw / bf16_peak,
            "note": "grad_w includes the activation quantization and both transposes"}


# LLaMA-70B-style layer matrices (out x in) and how many of each one layer holds; 80 layers.
WQ_70B_SHAPES = [(8192, 8192, 2), (1024, 8192, 2), (28672, 8192, 3)]
WQ_70B_LAYERS = 80


def weight_quant_figures(bl, device, hbm_peak: float):
    """bitlinear_quantize_weights on every 70B-shaped layer matrix (fp32 W ~ N(0, 0.015)),
    timed per shape over rotated copies, then totalled over 80 layers."""
    rows, total_ms, total_bytes = [], 0.0, 0
    for N, K, count in WQ_70B_SHAPES:
        n_bytes = N * K * 4
        copies = max(2, math.ceil(2 * L2_BYTES / n_bytes))
        Ws = [syn.weights(N, K, 0.015, seed=5000 + N + i, device=device) for i in range(copies)]
        packed = torch.empty((N, K // 4), dtype=torch.uint8, device=device)
        gamma = torch.empty(1, dtype=torch.float32, device=device)
        work = bl.workspace(1, N, K, device)
        calls = [(lambda W=W: bl.quantize_weights(W, EPS, packed=packed, gamma=gamma, ws=work))
                 for W in Ws]
        calls[0]()
        torch.cuda.synchronize()
        ms = time_back_to_back(calls, reps=3)
        alg = n_bytes + N * K // 4
        gbs = alg / (ms * 1e-3) / 1e9
        rows.append({"shape": f"{N}x{K}", "per_layer": count, "ms": ms, "GBps": gbs,
                     "frac_hbm": gbs / hbm_peak, "copies": copies})
        total_ms += ms * count * WQ_70B_LAYERS
        total_bytes += alg * count * WQ_70B_LAYERS
        del Ws, calls
        torch.cuda.empty_cache()
    gbs = total_bytes / (total_ms * 1e-3) / 1e9
    return {"shapes": rows, "all_layers": {"layers": WQ_70B_LAYERS, "ms": total_ms,
                                           "algorithmic_GB": total_bytes / 1e9, "GBps": gbs,
                                           "frac_hbm": gbs / hbm_peak,
                                           "note": "sum over shapes of per-matrix time x count"}}


# ----------------------------------------------------------------------------- main


DECODE_SHAPES = [("70b_up_8192x28672", 1), ("70b_up_8192x28672", 16), ("70b_up_8192x28672", 176),
                 ("70b_down_28672x8192", 1), ("70b_down_28672x8192", 16),
                 ("70b_down_28672x8192", 176), ("700m_up_1536x4096", 1),
                 ("700m_up_1536x4096", 4), ("700m_up_1536x4096", 16)]
BASE3_SHAPES = [("70b_up_8192x28672", 1), ("70b_down_28672x8192", 1), ("70b_up_8192x28672", 4),
                ("700m_up_1536x4096", 1)]


def secondary(bl, which: str, device):
    """One secondary figure (all of them for the headline line's roofline.others)."""
    hbm_peak, bf16_peak, _, _ = peaks()
    i8_peak = 2.0 * bf16_peak
    if which == "decode":
        return [decode_figure(bl, n, m, device, hbm_peak, i8_peak) for n, m in DECODE_SHAPES]
    if which == "decode_base3":
        return [decode3_figure(bl, n, m, device, hbm_peak) for n, m in BASE3_SHAPES]
    if which == "weight_quant":
        return weight_quant_figures(bl, device, hbm_peak)
    if which == "sweep":
        return sweep_3b_figures(bl, device, hbm_peak)
    if which == "backward":
        return backward_figure(bl, device, bf16_peak)
    raise ValueError(which)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return

    import ternary_weight_linear_03_b200 as bl

    if args.figure != "headline":
        if not torch.cuda.is_available():
            raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
        device = torch.device("cuda", 0)
        torch.cuda.set_device(device)
        print(json.dumps({"figure": args.figure, "result": secondary(bl, args.figure, device)}))
        return

    rank, world, local = bldist.rank_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    name, M = args.workload, args.M
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    hbm_peak, bf16_peak, _, peak_kind = peaks()
    i8_peak = 2.0 * bf16_peak  # nominal int8:bf16 dense ratio of 2 on the measured bf16 burst

    # Inputs of consecutive steps rotate over `copies` weight and activation copies, more
    # than twice L2 in total, so every step reads its operands from HBM (no L2 flush).
    step_bytes = N * K // 4 + M * K * (2 if wl["x_dtype"] == torch.bfloat16 else 4)
    copies = max(2, math.ceil(2 * L2_BYTES / step_bytes))
    off = bldist.seed_offset(rank)
    ws_copies = packed_copies(bl, name, device, copies, seed_offset=off)
    xs = act_copies(name, M, device, copies, seed_offset=off)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    work = bl.workspace(M, N, K, device)
    stream = torch.cuda.current_stream()

    def step(i):
        packed, gamma = ws_copies[i % copies]
        bl.forward(xs[i % copies], packed, gamma, y=y, ws=work)

    for i in range(max(args.warmup, 2)):  # eager warm-up also configures every kernel
        step(i)
    torch.cuda.synchronize()
    assert bl.get_device_status() == 0

    # One CUDA graph per copy holding that step's forward; the timed loop replays them in
    # turn, one graph per step.
    graphs = []
    for i in range(copies):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(i)
        graphs.append(g)
    for i in range(max(3, args.warmup)):
        graphs[i % copies].replay()
    torch.cuda.synchronize()
    assert bl.get_device_status() == 0

    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        start.record(stream)
        for i in range(args.steps):
            graphs[i % copies].replay()
        end.record(stream)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    elapsed_ms = bldist.max_over_ranks(start.elapsed_time(end), dist, device)
    status = bl.get_device_status()
    if status != 0:
        raise SystemExit(f"device status {bl.status_string(status)} after the timed region")
    del graphs
    tokens = M * args.steps * world
    value = tokens / (elapsed_ms * 1e-3)

    # end to end through the public API with host buffers (pinned): every step, the batch
    # goes up, the forward runs on the resident packed weights and the output comes back.
    # Three streams and two buffers of each kind: the upload of step i + 1 and the download
    # of step i - 1 run while the forward of step i computes (PCIe is full duplex, with a
    # copy engine per direction), as a serving loop would overlap them.
    e2e = None
    if not args.no_e2e:
        x_h = xs[0].cpu().pin_memory()
        y_hs = [torch.empty((M, N), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        x_ds = [torch.empty_like(xs[0]) for _ in range(2)]
        y_ds = [y, torch.empty_like(y)]
        packed, gamma = ws_copies[0]
        e2e_steps = max(3, min(args.steps, 20))
        s_in = torch.cuda.Stream(device)
        s_out = torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_comp = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i % 2
            s_in.wait_event(ev_comp[b])  # the forward two steps back has read x_ds[b]
            with torch.cuda.stream(s_in):
                x_ds[b].copy_(x_h, non_blocking=True)
            ev_in[b].record(s_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])  # y_ds[b] of two steps back is home
            bl.forward(x_ds[b], packed, gamma, y=y_ds[b], ws=work, stream=stream)
            ev_comp[b].record(stream)
            s_out.wait_event(ev_comp[b])
            with torch.cuda.stream(s_out):
                y_hs[b].copy_(y_ds[b], non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        s2 = torch.cuda.Event(enable_timing=True)
        e2 = torch.cuda.Event(enable_timing=True)
        s2.record(s_in)
        for i in range(e2e_steps):
            e2e_step(i)
        s_in.wait_stream(s_out)  # the last download is part of the step
        e2.record(s_in)
        torch.cuda.synchronize()
        e_ms = bldist.max_over_ranks(s2.elapsed_time(e2), dist, device)
        e2e = {"value": M * e2e_steps * world / (e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": x_h.numel() * x_h.element_size(),
               "d2h_bytes_per_step": y_hs[0].numel() * y_hs[0].element_size(),
               "steps": e2e_steps, "overlap": "upload, forward and download on three streams"}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    # ------------------------------------------------------------------ roofline
    # One step is one bitlinear_forward call (its kernels back to back), so the launch time
    # is the timed region's average step.
    fw_ms = elapsed_ms / args.steps
    path, splits = bl.debug_plan(M, N, K)
    fw_ops = 2.0 * M * N * K
    fw_bytes = N * K // 4 + M * K * 2 + M * N * 2
    if path == "prefill":
        # the activation quantization of the same batch timed alone, for the GEMM's share
        xq_calls = [(lambda i=i: bl.quantize_acts(xs[i])) for i in range(min(copies, 4))]
        xq_calls[0]()
        aq_ms = time_back_to_back(xq_calls)
        achieved = fw_ops / (fw_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": i8_peak, "unit": "TFLOP/s",
                    "frac": achieved / i8_peak,
                    "traffic": ncu_traffic("gemm_prefill_kernel", name, M),
                    "peak_source": f"{peak_kind} bf16 burst x 2 (int8 ops, nominal ratio)",
                    "kernel": "bitlinear_forward = act_quant_kernel + gemm_prefill_kernel "
                              "(tcgen05 kind::i8, weights in TMEM)",
                    "algorithmic_ops_per_launch": fw_ops, "ms_per_launch": fw_ms,
                    "act_quant_ms": aq_ms, "gemm_ms_est": fw_ms - aq_ms,
                    "gemm_frac_est": fw_ops / ((fw_ms - aq_ms) * 1e-3) / 1e12 / i8_peak}
    else:
        achieved = fw_bytes / (fw_ms * 1e-3) / 1e9
        kern = "gemv_kernel" if path == "gemv" else "gemm_skinny_kernel"
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak, "traffic": ncu_traffic(kern, name, M),
                    "peak_source": f"{peak_kind} HBM copy", "kernel": f"bitlinear_forward ({path})",
                    "algorithmic_bytes_per_launch": fw_bytes, "ms_per_launch": fw_ms}

    others = {}
    if not args.no_others:
        others["decode"] = secondary(bl, "decode", device)
        others["decode_base3"] = secondary(bl, "decode_base3", device)
        others["weight_quant_70b"] = secondary(bl, "weight_quant", device)
        others["sweep_3b_26_layers"] = secondary(bl, "sweep", device)
        others["backward_ste"] = secondary(bl, "backward", device)
    roofline["others"] = others

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(name, M)
    config = config_of(name, M, wl, world)
    config["inputs_vs_l2"] = (f"{copies} copies of packed W + x rotated "
                              f"({copies * step_bytes / 2**20:.0f} MiB > 2 x L2), no flush")
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8xternary->i32 (bf16 in/out)", "data": "synthetic", "config": config,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.result(),
        "gpu_launches": forward_launches(bl, M, N, K) * args.steps,
    }
    print(json.dumps(out))


if __name__ == "__main__":
    main()
