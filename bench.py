#!/usr/bin/env python3
"""BitLinear forward benchmark on B200: one JSON line per run (rank 0).

A step is one pass of the whole BitLinear hot path over one batch: absmean ternary
quantization of the fp32 weight matrix (gamma, codes, 2-bit packing), per-token int8
quantization of the activations, the int32 contraction and the rescale to bf16.

The timed loop replays one CUDA graph per step (captured from the same library calls), so
host launch overhead is not part of the number; `e2e` times the plain library calls with
host buffers instead.

Default workload: the 700M-class FFN up-projection (K=1536, N=4096, W ~ N(0, 0.02) fp32,
bf16 activations ~ N(0, 1) with 1% outlier channels x20), M = 16 tokens. Inputs larger
than L2: the step cycles through enough weight copies (8 x 25 MB) that every step reads
its weights from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--M M]

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


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=10)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="700m_up_1536x4096")
    p.add_argument("--M", type=int, default=16)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    return p.parse_args()


KERNEL_SOURCES = {"weight_quant_kernel": "weight_quant.cuh", "gemm_tc_kernel": "gemm_tc.cuh",
                  "gemm_skinny_kernel": "gemm_skinny.cuh", "gemv_kernel": "gemv.cuh"}


def ncu_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when the
    capture was of another workload or the kernel source changed since it was taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "ternary_weight_linear_03_b200", "csrc", KERNEL_SOURCES[kernel])
    try:
        rec = json.load(open(path))[kernel]
        sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("workload") != workload or rec.get("source_sha1") != sha:
        return None
    return rec["dram_bytes_per_launch"]


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


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


# ----------------------------------------------------------------------------- workload


def make_inputs(name: str, M: int, device, copies: int, seed_offset: int = 0):
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    Ws = [syn.weights(N, K, wl["sigma"], seed=syn.w_seed(name, i) + seed_offset).to(device)
          for i in range(copies)]
    xs = [syn.activations(M, K, seed=syn.x_seed(name, M) + 97 * i + seed_offset,
                          dtype=wl["x_dtype"], outlier_frac=wl["outlier_frac"]).to(device)
          for i in range(copies)]
    return N, K, Ws, xs


def cpu_baseline(name: str, M: int, budget_s: float = 12.0):
    """The oracle, as it stands, on this host: quantize W and run the forward for M tokens,
    repeated until budget_s has passed (the whole workload per step)."""
    from oracle import oracle as orc
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    W = syn.weights(N, K, wl["sigma"], seed=syn.w_seed(name)).numpy()
    x = syn.activations(M, K, seed=syn.x_seed(name, M), dtype=wl["x_dtype"],
                        outlier_frac=wl["outlier_frac"])
    xin = syn.bf16_bits(x) if x.dtype == torch.bfloat16 else x.numpy()
    steps, t0 = 0, time.perf_counter()
    while True:
        packed, gamma = orc.quantize_weights(W, 1e-5)
        orc.forward(xin, packed, gamma, out="bf16")
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": M * steps / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{steps} full steps ({name}, M={M}: quantize W {N}x{K} fp32 + forward),"
                      f" single-threaded C++ oracle, {el:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from oracle import oracle as orc
    name, M = args.workload, args.M
    wl = syn.WORKLOADS[name]
    N, K = wl["N"], wl["K"]
    W = syn.weights(N, K, wl["sigma"], seed=syn.w_seed(name)).numpy()
    x = syn.activations(M, K, seed=syn.x_seed(name, M), dtype=wl["x_dtype"],
                        outlier_frac=wl["outlier_frac"])
    xin = syn.bf16_bits(x) if x.dtype == torch.bfloat16 else x.numpy()
    # A bounded sample per step: the first R weight rows go through the whole path
    # (absmean over those rows, ternarize, pack, forward for all M tokens). Every part of
    # the work is linear in the number of rows, so tokens/s = M * R / (N * step time).
    R = min(N, 512)
    Wr = np.ascontiguousarray(W[:R])

    def step():
        packed, gamma = orc.quantize_weights(Wr, 1e-5)
        orc.forward(xin, packed, gamma, out="bf16")

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    value = M * args.steps * R / (N * el)
    sample = (f"each step: rows 0..{R - 1} of the {N}x{K} weights through absmean, ternarize, "
              f"pack and the forward of M={M} tokens; scaled by {R}/{N} (work is linear in rows)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8/i32 (fp32 quantization)", "data": "synthetic",
        "config": {"workload": name, "M": M, "N": N, "K": K},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
        return

    import ternary_weight_linear_03_b200 as bl

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
    w_bytes = N * K * 4
    copies = max(2, math.ceil(2 * L2_BYTES / w_bytes))
    N, K, Ws, xs = make_inputs(name, M, device, copies, seed_offset=bldist.seed_offset(rank))
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device=device)
    gamma = torch.empty(1, dtype=torch.float32, device=device)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    ws = bl.workspace(M, N, K, device)
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        if ev is not None:
            ev[0].record()
        bl.quantize_weights(Ws[i % copies], 1e-5, packed=packed, gamma=gamma, ws=ws)
        if ev is not None:
            ev[1].record()
        bl.forward(xs[i % copies], packed, gamma, y=y, ws=ws)
        if ev is not None:
            ev[2].record()

    for i in range(max(args.warmup, copies)):  # eager warm-up also configures every kernel
        step(i)
    torch.cuda.synchronize()
    assert bl.get_device_status() == 0

    # One CUDA graph per weight copy (the step's launches with timing-event nodes between
    # the weight quantization and the forward); the timed loop replays them in turn.
    graphs, evs = [], []
    for i in range(copies):
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(i, ev)
        graphs.append(g)
        evs.append(ev)
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

    # per-launch times: the event nodes of each copy's graph as of its last replay
    wq_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    fw_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    hbm_peak, bf16_peak, peak_kind = peaks()
    wq_bytes = N * K * 4 + N * K // 4
    fw_bytes = N * K // 4 + M * K * 2 + M * N * 2
    fw_ops = 2.0 * M * N * K
    others = {"quantize_weights_ms": wq_ms, "forward_ms": fw_ms,
              "forward_GBps": fw_bytes / (fw_ms * 1e-3) / 1e9,
              "forward_TOPS": fw_ops / (fw_ms * 1e-3) / 1e12}
    if wq_ms >= fw_ms:
        achieved = wq_bytes / (wq_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak,
                    "traffic": ncu_traffic("weight_quant_kernel", name),
                    "peak_source": f"{peak_kind} HBM copy",
                    "kernel": "bitlinear_quantize_weights (absmean + ternarize/pack)",
                    "algorithmic_bytes": wq_bytes, "ms_per_launch": wq_ms}
    elif M > 256:
        # the tcgen05 int8 GEMM: a dense contraction, measured against the int8 tensor peak
        # (the measured bf16 burst figure times the nominal int8:bf16 ratio of 2)
        i8_peak = 2.0 * bf16_peak
        achieved = fw_ops / (fw_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": i8_peak, "unit": "TFLOP/s",
                    "frac": achieved / i8_peak, "traffic": ncu_traffic("gemm_tc_kernel", name),
                    "peak_source": f"{peak_kind} bf16 burst x 2 (int8)",
                    "kernel": "bitlinear_forward (activation quant + tcgen05 int8 GEMM)",
                    "algorithmic_ops": fw_ops, "ms_per_launch": fw_ms}
    else:
        achieved = fw_bytes / (fw_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                    "frac": achieved / hbm_peak, "traffic": None,
                    "peak_source": f"{peak_kind} HBM copy", "kernel": "bitlinear_forward",
                    "algorithmic_bytes": fw_bytes, "ms_per_launch": fw_ms}
    roofline["others"] = others

    tokens = M * args.steps * world
    value = tokens / (elapsed_ms * 1e-3)

    # end to end through the public API with host buffers (pinned), H2D + D2H timed
    e2e = None
    if not args.no_e2e:
        W_h = Ws[0].cpu().pin_memory()
        x_h = xs[0].cpu().pin_memory()
        y_h = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        W_d = torch.empty_like(Ws[0])
        x_d = torch.empty_like(xs[0])
        e2e_steps = max(3, min(args.steps, 50))
        for _ in range(2):
            W_d.copy_(W_h, non_blocking=True)
            x_d.copy_(x_h, non_blocking=True)
            bl.quantize_weights(W_d, 1e-5, packed=packed, gamma=gamma, ws=ws)
            bl.forward(x_d, packed, gamma, y=y, ws=ws)
            y_h.copy_(y, non_blocking=True)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        s2 = torch.cuda.Event(enable_timing=True)
        e2 = torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for _ in range(e2e_steps):
            W_d.copy_(W_h, non_blocking=True)
            x_d.copy_(x_h, non_blocking=True)
            bl.quantize_weights(W_d, 1e-5, packed=packed, gamma=gamma, ws=ws)
            bl.forward(x_d, packed, gamma, y=y, ws=ws)
            y_h.copy_(y, non_blocking=True)
        e2.record(stream)
        torch.cuda.synchronize()
        e_ms = bldist.max_over_ranks(s2.elapsed_time(e2), dist, device)
        e2e = {"value": M * e2e_steps * world / (e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": W_h.numel() * 4 + x_h.numel() * x_h.element_size(),
               "d2h_bytes_per_step": y_h.numel() * 2, "steps": e2e_steps}

    del graphs
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(name, M)
    launches_per_step = 1 + (1 if M <= 4 else 2)  # weight quant + (GEMV | act quant + GEMM)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "i8xternary->i32 (fp32 quantization, bf16 out)", "data": "synthetic",
        "config": {"workload": name, "M": M, "N": N, "K": K, "w_dtype": "fp32",
                   "x_dtype": str(wl["x_dtype"]).replace("torch.", ""), "out": "bf16",
                   "inputs_vs_l2": f"{copies} weight copies x {w_bytes / 2**20:.1f} MiB rotated "
                                   f"(> L2), no flush", "parallelism": f"replicas x{world}"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "clocks": clk.result(),
        "gpu_launches": launches_per_step * args.steps,
    }
    print(json.dumps(out))


if __name__ == "__main__":
    main()
