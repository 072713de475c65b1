#!/usr/bin/env python
"""Throughput of the fused SignRot online path (rotate + sign-adjust + asymmetric INT4 quant).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config 4] [--also 3]

One step = one pass of the online path over the workload's T tokens resident in HBM
(signrot_rotate_quant on [T, n] bf16 rows -> packed INT4 codes + fp32 scale/zero). The default
workload is LLaMA-3-70B's down projection (n = 28672, T = 16384 per GPU), the largest one that
fits one GPU; LLaMA-3-8B's (n = 14336, T = 8192) is measured the same way and reported under
"also". The outlier channel and sign vector come from a calibration pass (signrot_calibrate +
signrot_build_sign) run once before timing; its time is reported separately under
"calibration". Multi-GPU runs shard tokens (weak scaling: every rank processes its own T tokens,
no data-path collective).

Rank 0 prints one JSON line. --impl reference times the float64 CPU oracle on a bounded sample
of the same workload (a reported CPU baseline). --quant picks another grid of the same kernels;
--sweep measures the decode/prefill T sweep and the long calibration pass at n = 14336.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from rotation_activation_quantization_b200 import sharding  # noqa: E402
from rotation_activation_quantization_b200 import synthetic as syn  # noqa: E402

METRIC = "tokens/s and achieved HBM GB/s (% of B200 peak) for fused rotate+INT4 quant"
UNIT = "tokens/s"
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=4,
                    help="workload index (1..6); 4 = LLaMA3-70B down_proj (n = 28672, the largest single-GPU "
                         "workload), 3 = LLaMA3-8B (n = 14336), 6 = LLaMA2-7B (n = 11008)")
    ap.add_argument("--also", type=lambda v: [int(i) for i in v.split(",") if i], default=None,
                    help="comma-separated workloads measured the same way and reported under 'also' "
                         "(default: 3 beside the default workload, none otherwise)")
    ap.add_argument("--tokens", type=int, default=None, help="override tokens per GPU")
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-oracle sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-gemm", action="store_true",
                    help="skip the W4A4 down-projection measurement reported under consumer_gemm")
    ap.add_argument("--quant", choices=["asym4", "asym8", "sym4", "sym8"], default="asym4",
                    help="grid of the timed kernel: asymmetric INT4 (the metric's), INT8, or symmetric")
    ap.add_argument("--calib-tokens", type=int, default=None,
                    help="--sweep: calibration tokens (default 128 x 2048; a multiple of 2048)")
    ap.add_argument("--sweep", action="store_true",
                    help="decode/prefill sweep at n = 14336 (T = 1 .. 32768, latency per call and GB/s, "
                         "warm and after an L2 flush) and the 128 x 2048-token calibration pass; one GPU")
    return ap.parse_args(argv)


def _default_also(args) -> None:
    if args.also is None:
        args.also = [3] if (args.config == 4 and not args.tokens) else []


def workload(args) -> syn.Workload:
    w = syn.workload(args.config)
    return w.with_T(args.tokens) if args.tokens else w


def bytes_per_token(w: syn.Workload, quant: str = "asym4") -> int:
    """Algorithmic HBM bytes per token: activations in, codes out (packed two per byte for 4 bits,
    one per byte for 8), fp32 scale (+ fp32 zero-point on the asymmetric grid)."""
    bits = 8 if quant.endswith("8") else 4
    return w.in_bytes * w.n + w.n * bits // 8 + (4 if quant.startswith("sym") else 8)


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return {"hbm_gbs": float(json.load(f)["hbm_gbs"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "source": "fallback"}


# the fused kernels' translation unit and every header it includes
FUSED_SOURCES = ("rotate_tc.cu", "signrot_device.cuh", "signrot_internal.h", "tc_ptx.cuh")


def kernel_sources_digest() -> str:
    """Digest of the fused kernels' sources: a recorded ncu traffic figure applies while it holds."""
    csrc = os.path.join(ROOT, "rotation_activation_quantization_b200", "csrc")
    h = hashlib.sha256()
    for f in FUSED_SOURCES:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(w: syn.Workload, digest: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on these sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    e = rec.get(w.name)
    if not e or e.get("kernel_sources") != digest:
        return None
    return float(e["dram_bytes_per_token"]) * w.T


def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = max((i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"), default=0)
        if n:
            return int(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_sample(w: syn.Workload, seconds: float, tokens_per_call: int = 8, fast: bool = False):
    """Time the CPU oracle (float64 dense rotation + fp32 quantizer; with ``fast`` its O(n log n)
    cross-check form instead) on token blocks until the budget is spent. The rows are drawn before
    the clock starts. Returns (tokens/s, tokens, seconds)."""
    from oracle import signrot_oracle as o

    d = syn.draw_d(w)
    xc = o.to_f64(syn.draw_calibration(w, 0, min(256, syn.calibration_size(w))), w.dtype)
    k, xk = o.calibrate(xc)
    s = o.build_sign(w.n, k, xk, d)
    pool = o.to_f64(syn.draw_tokens(w, 0, min(w.T, 256)), w.dtype)
    done, t0 = 0, time.perf_counter()
    while True:
        i = done % (pool.shape[0] - tokens_per_call + 1)
        x = pool[i:i + tokens_per_call]
        if fast:
            o.quantize_asym(o.rotate_fast(x, d, s))
        else:
            o.rotate_quant(x, d, s)
        done += x.shape[0]
        el = time.perf_counter() - t0
        if el >= seconds:
            return done / el, done, el


class ClockSampler:
    """Polls NVML (the source nvidia-smi reads) for SM clock, power and throttle reasons while
    the timed region runs."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz, self.err = [], 0, None, None
        self._stop = threading.Event()
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        except Exception as e:  # clocks are reported as unavailable, never invented
            self.h, self.err = None, f"{type(e).__name__}: {e}"

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception as e:
                self.err = f"{type(e).__name__}: {e}"
                return
            time.sleep(0.0005)

    def __enter__(self):
        if self.h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.h is not None:
            self._t.join(timeout=2)

    def report(self) -> dict:
        if self.h is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.err or "no samples"}
        reasons = [name for bit, name in self.REASONS.items() if self.reasons & bit]
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


def run_reference(args) -> int:
    """The reference arm: the float64 oracle on the host cores, exactly K timed steps after W
    untimed ones, each step a sample of the workload's rows sized so the run stays within a few
    minutes (1 to 4 tokens per step)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = workload(args)
    cores = cpu_cores()
    from oracle import signrot_oracle as o

    d = syn.draw_d(w)
    xc = o.to_f64(syn.draw_calibration(w, 0, min(256, syn.calibration_size(w))), w.dtype)
    k, xk = o.calibrate(xc)
    s = o.build_sign(w.n, k, xk, d)
    xs = o.to_f64(syn.draw_tokens(w, 0, 4), w.dtype)
    o.rotate_quant(xs[:1], d, s)  # builds and caches the dense H
    t0 = time.perf_counter()
    o.rotate_quant(xs[:1], d, s)
    per_token = max(time.perf_counter() - t0, 1e-6)
    budget = 150.0
    K, W = max(args.steps, 1), max(args.warmup, 0)
    tokens_per_step = int(max(1, min(4, budget / ((K + W) * per_token))))
    xs = xs[:tokens_per_step]
    for _ in range(W):
        o.rotate_quant(xs, d, s)
    t0 = time.perf_counter()
    for _ in range(K):
        o.rotate_quant(xs, d, s)
    el = time.perf_counter() - t0
    value = tokens_per_step * K / el
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": K, "warmup": W, "ms_per_step": 1e3 * el / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "n": w.n, "tokens_per_step": tokens_per_step,
                   "input_dtype": w.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"{tokens_per_step} tokens of {w.name} per step, dense float64 "
                                   f"O(n^2) rotation + fp32 quantizer"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def _to_dev(torch, a: np.ndarray, dtype: str, dev):
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def measure_kernel(torch, sr, w: syn.Workload, args, dev, world: int, rank: int, quant: str) -> dict:
    """Device time of K launches of the fused call over this rank's T tokens of workload w.

    Inputs larger than L2: K back-to-back launches between one event pair (an event recorded
    between two launches would also stop the next launch from being scheduled while the previous
    one drains). Inputs that fit in L2: each launch timed alone by its own event pair after a
    write larger than L2 (flushed), and the K launches back to back as well (warm, reported
    beside it)."""
    import torch.distributed as dist

    T, n = w.T, w.n
    x_np = syn.draw_tokens(w, *sharding.weak_shard(rank, T))
    d_np = syn.draw_d(w)
    xc_np = syn.draw_calibration(w)
    x = _to_dev(torch, x_np, w.dtype, dev)
    d = torch.from_numpy(d_np).to(dev)
    stream = torch.cuda.current_stream(dev)

    # calibration (once per model; timed on its own)
    xc = _to_dev(torch, xc_np, w.dtype, dev)
    ws = torch.empty(n, dtype=torch.int64, device=dev)
    for _ in range(2):
        k, xk, _ = sr.calibrate(xc, ws=ws)
        s = sr.build_sign(n, k, xk, d)
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    k, xk, _ = sr.calibrate(xc, ws=ws)
    s = sr.build_sign(n, k, xk, d)
    c1.record(stream)
    torch.cuda.synchronize(dev)
    calib_ms = c0.elapsed_time(c1)
    del xc, s

    bits = 8 if quant.endswith("8") else 4
    sym = quant.startswith("sym")
    q = torch.empty((T, n * bits // 8), dtype=torch.int8 if (sym and bits == 8) else torch.uint8, device=dev)
    scale = torch.empty(T, dtype=torch.float32, device=dev)
    zero = torch.empty(T, dtype=torch.float32, device=dev)

    def step():
        if sym:
            sr.rotate_quant_sym_outlier(x, d, k, xk, bits=bits, q=q, scale=scale)
        else:
            sr.rotate_quant_outlier(x, d, k, xk, bits=bits, q=q, scale=scale, zero=zero)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)

    K = args.steps
    bpt = bytes_per_token(w, quant)
    resident = T * bpt < 2 * L2_BYTES
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev) if resident else None
    sampler = ClockSampler(dev.index)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = sr.kernel_launches()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with sampler:
        if resident:
            ms = 0.0
            for _ in range(K):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                step()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                ms += e0.elapsed_time(e1)
            region_ms = ms
        else:
            ev0.record(stream)
            for _ in range(K):
                step()
            ev1.record(stream)
            torch.cuda.synchronize(dev)
            region_ms = ev0.elapsed_time(ev1)
    launches = sr.kernel_launches() - launches0
    warm_ms = None
    if resident:  # the same launches back to back with the inputs left in L2
        ev0.record(stream)
        for _ in range(K):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        warm_ms = ev0.elapsed_time(ev1)
    if world > 1:
        dist.barrier()
    region_ms_max = sharding.max_over_ranks(region_ms, device=dev)
    avg_launch_ms = region_ms / K  # the fused kernel is the only launch in the region
    achieved = bpt * T / (avg_launch_ms * 1e-3) / 1e9
    return {"w": w, "x_np": x_np, "x": x, "d": d, "k": k, "xk": xk, "region_ms": region_ms,
            "region_ms_max": region_ms_max, "avg_launch_ms": avg_launch_ms, "achieved": achieved, "bpt": bpt,
            "launches": launches, "calib_ms": calib_ms, "calib_tokens": int(xc_np.shape[0]), "sampler": sampler,
            "resident": resident, "warm_ms": warm_ms, "sym": sym}


# The down projection each workload's activations feed: (K = n, N = the model's hidden size).
GEMM_SHAPES = {3: (14336, 4096), 4: (28672, 8192), 5: (14336, 4096), 6: (11008, 4096)}


def int8_peak_tops() -> tuple[float, str]:
    """Dense int8 tensor peak: the measured bf16 GEMM rate (burst) times the nominal int8/bf16
    ratio of B200 (4.5 / 2.25 = 2)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 2 (nominal int8/bf16 ratio)"
    return 2.0 * 1590.0, "fallback bf16 1.59 PFLOP/s x 2 (nominal int8/bf16 ratio)"


def measure_gemm(torch, sr, T: int, K: int, N: int, dev, steps: int, warmup: int) -> dict:
    """The W4A4 down projection (signrot_w4a4_matmul) on random codes of the workload's shape:
    device time of `steps` back-to-back launches; the operands (T x K / 2 + N x K bytes) exceed L2."""
    g = torch.Generator(device=dev).manual_seed(1234)
    q = torch.randint(0, 256, (T, K // 2), dtype=torch.uint8, device=dev, generator=g)
    wq4 = torch.randint(0, 256, (N, K // 2), dtype=torch.uint8, device=dev, generator=g)
    scale = torch.rand(T, device=dev, generator=g) * 0.1 + 0.01
    zero = torch.randint(-100, 20, (T,), device=dev, generator=g).float()
    wscale = torch.rand(N, device=dev, generator=g) * 0.01 + 1e-3
    wq8, colsum = sr.w4a4_prepare_weights(wq4, K)
    out = torch.empty((T, N), dtype=torch.float32, device=dev)
    for _ in range(warmup):
        sr.w4a4_matmul(q, scale, zero, wq8, wscale, colsum, out=out)
    torch.cuda.synchronize(dev)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    l0 = sr.kernel_launches()
    e0.record(stream)
    for _ in range(steps):
        sr.w4a4_matmul(q, scale, zero, wq8, wscale, colsum, out=out)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1) / steps
    tops = 2.0 * T * N * K / (ms * 1e-3) / 1e12
    peak, src = int8_peak_tops()
    return {"call": "signrot_w4a4_matmul", "T": T, "K": K, "N": N, "ms_per_launch": ms,
            "tokens_per_s": T / (ms * 1e-3), "launches": sr.kernel_launches() - l0, "steps": steps,
            "roofline": {"bound": "tensor", "achieved": tops, "peak": peak, "unit": "TOPS (int8)",
                         "frac": tops / peak, "peak_source": src, "ops_per_launch": 2.0 * T * N * K}}


def roofline_entry(m: dict, quant: str, peaks: dict, digest: str) -> dict:
    w = m["w"]
    traffic = recorded_traffic(w, digest) if quant == "asym4" else None
    return {"bound": "hbm", "achieved": m["achieved"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": m["achieved"] / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peaks["source"],
            "frac_of_nominal_8tbs": m["achieved"] / NOMINAL_HBM_GBS,
            "bytes_per_token": m["bpt"], "tokens_per_launch": w.T,
            "kernel": "signrot_rotate_quant" if not m["sym"] else "signrot_rotate_quant_sym",
            "kernel_sources": digest, "launch_ms_mean": m["avg_launch_ms"]}


def l2_note(m: dict) -> str:
    mb = m["bpt"] * m["w"].T / 1e6
    if m["resident"]:
        return (f"inputs fit in L2 ({mb:.1f} MB per step vs {L2_BYTES / 1e6:.0f} MB): each launch timed "
                f"alone after a {2 * L2_BYTES / 1e6:.0f} MB L2-flushing write; warm back-to-back rate beside it")
    return f"inputs larger than L2 ({mb:.1f} MB per step vs {L2_BYTES / 1e6:.0f} MB), no flush"


def run_ours(args) -> int:
    import torch
    import torch.distributed as dist

    from rotation_activation_quantization_b200 import signrot as sr

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta

        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=dev)
    sr.lib()
    stream = torch.cuda.current_stream(dev)

    w = workload(args)
    T, n = w.T, w.n
    m = measure_kernel(torch, sr, w, args, dev, world, rank, args.quant)
    x_np, d, k, xk = m["x_np"], m["d"], m["k"], m["xk"]
    h2d = m["x"].numel() * m["x"].element_size()
    del m["x"]

    # end to end through the host-buffer C-ABI call: pinned host rows -> HBM -> fused kernel ->
    # pinned host codes, chunked over two streams so copies overlap (the copies are timed)
    E = args.e2e_steps or max(3, min(args.steps, 20))
    xh = torch.from_numpy(x_np.view(np.int16)).view(torch.bfloat16) if w.dtype == "bf16" else torch.from_numpy(x_np)
    xh = xh.pin_memory()
    qh = torch.empty((T, n // 2), dtype=torch.uint8).pin_memory()
    sh = torch.empty(T, dtype=torch.float32).pin_memory()
    zh = torch.empty(T, dtype=torch.float32).pin_memory()
    chunk = min(T, 1024)
    wsb = torch.empty(2 * (chunk * sr.host_bytes_per_token(n, xh.dtype) + 64), dtype=torch.uint8, device=dev)

    def e2e_step():
        sr.rotate_quant_host(xh, d, qh, sh, zh, wsb, k=k, xk=xk, device=dev)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sharding.max_over_ranks(e0.elapsed_time(e1), device=dev)
    if world > 1:
        dist.barrier()
    d2h = qh.numel() + 4 * sh.numel() + 4 * zh.numel()
    del xh, qh, sh, zh, wsb

    # companion workloads, same kernel family, device-timed the same way (one line, extra keys)
    companions = {}
    for ci in args.also:
        if ci == args.config:
            continue
        mc = measure_kernel(torch, sr, syn.workload(ci), args, dev, world, rank, args.quant)
        del mc["x"]
        companions[ci] = mc

    gemm = None
    if args.config in GEMM_SHAPES and not args.no_gemm:
        Kg, Ng = GEMM_SHAPES[args.config]
        gemm = measure_gemm(torch, sr, T, Kg, Ng, dev, max(3, min(args.steps, 20)), 3)

    if rank == 0:
        peaks = measured_peaks()
        digest = kernel_sources_digest()
        K = args.steps
        value = sharding.aggregate_rate(world * T * K, m["region_ms_max"] * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": m["region_ms_max"] / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {
                "workload": w.name, "n": n, "tokens_per_gpu": T, "global_tokens": world * T,
                "input_dtype": w.dtype, "quant": args.quant,
                "output": {"asym4": "INT4 packed [T, n/2] + fp32 scale/zero [T]",
                           "asym8": "INT8 [T, n] + fp32 scale/zero [T]",
                           "sym4": "signed INT4 packed [T, n/2] + fp32 scale [T]",
                           "sym8": "int8 [T, n] + fp32 scale [T]"}[args.quant],
                "parallelism": f"token-sharded x{world} (no collective)",
                "l2": l2_note(m),
            },
            "hbm_gbs": m["achieved"],
            "hbm_frac": m["achieved"] / peaks["hbm_gbs"],
            "roofline": roofline_entry(m, args.quant, peaks, digest),
            "e2e": {"value": world * T * E / (e2e_ms * 1e-3), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms / E, "steps": E,
                    "call": "signrot_rotate_quant_host (asymmetric INT4 grid)"},
            "gpu_launches": int(m["launches"]),
            "calibration": {"tokens": m["calib_tokens"], "ms": m["calib_ms"],
                            "gbs": m["calib_tokens"] * n * w.in_bytes / (m["calib_ms"] * 1e-3) / 1e9},
            "clocks": m["sampler"].report(),
        }
        if gemm is not None:
            line["consumer_gemm"] = gemm
        if m["warm_ms"] is not None:
            line["warm_l2"] = {"value": T * K / (m["warm_ms"] * 1e-3), "unit": UNIT,
                               "gbs": m["bpt"] * T * K / (m["warm_ms"] * 1e-3) / 1e9}
        if companions:
            line["also"] = {}
            for ci, mc in companions.items():
                wc = mc["w"]
                entry = {"workload": wc.name, "n": wc.n, "tokens_per_gpu": wc.T,
                         "value": world * wc.T * K / (mc["region_ms_max"] * 1e-3), "unit": UNIT,
                         "ms_per_step": mc["region_ms_max"] / K, "l2": l2_note(mc),
                         "roofline": roofline_entry(mc, args.quant, peaks, digest),
                         "gpu_launches": int(mc["launches"]), "clocks": mc["sampler"].report()}
                if mc["warm_ms"] is not None:
                    entry["warm_l2"] = {"value": wc.T * K / (mc["warm_ms"] * 1e-3), "unit": UNIT,
                                        "gbs": mc["bpt"] * wc.T * K / (mc["warm_ms"] * 1e-3) / 1e9}
                line["also"][wc.name] = entry
        if world == 1 and not args.no_cpu_baseline:
            v, done, el = oracle_sample(w, args.cpu_seconds)
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                                    "sample": f"{done} tokens of {w.name} in {el:.1f} s (float64 dense "
                                              f"O(n^2) rotation + fp32 quantizer)"}
            vf, donef, elf = oracle_sample(w, min(3.0, args.cpu_seconds), fast=True)
            line["cpu_fast_form"] = {"value": vf, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                                     "sample": f"{donef} tokens of {w.name} in {elf:.1f} s (the oracle's "
                                               f"O(n log n) cross-check form: H_F block + FWHT, float64)"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def graph_replay(torch, call, stream, dev, per_graph: int = 20, replays: int = 10) -> dict:
    """Device time per call with the host out of the loop: ``per_graph`` calls captured in one
    CUDA graph, replayed ``replays`` times between one event pair."""
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(per_graph):
                call()
        g.replay()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(replays):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        us = e0.elapsed_time(e1) * 1e3 / (per_graph * replays)
        del g
        return {"us_per_call_graph": us}
    except Exception as exc:  # reported, not fatal: the other rows stand
        return {"graph_error": f"{type(exc).__name__}: {exc}"[:200]}


def run_sweep(args) -> int:
    """Decode/prefill sweep of the fused call and the calibration pass over 128 x 2048 tokens.

    Rows: the first 8192 tokens of the sweep workload drawn on the host, tiled 4x on the device
    for T = 32768; calibration: its first 8192 calibration rows tiled 32x (262144 tokens, 7.5 GB).
    Tiling changes no work: every kernel here reads every row and does the same arithmetic on it.
    """
    import torch

    from rotation_activation_quantization_b200 import signrot as sr

    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
    if not torch.cuda.is_available():
        raise RuntimeError("bench.py needs a CUDA device")
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    sr.lib()
    w = syn.workload(5)
    n, Tmax = w.n, max(syn.SWEEP_T)
    base = 8192

    def bf(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)

    x = bf(syn.draw_tokens(w, 0, base)).repeat(Tmax // base, 1)
    d = torch.from_numpy(syn.draw_d(w)).to(dev)
    n_cal = args.calib_tokens or w.calib_T
    if n_cal <= 0 or n_cal % 2048:
        raise ValueError("--calib-tokens must be a positive multiple of 2048")
    xc = bf(syn.draw_calibration(w, 0, base)).repeat((n_cal + base - 1) // base, 1)[:n_cal]
    stream = torch.cuda.current_stream(dev)
    ws = torch.empty(n, dtype=torch.int64, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    peaks = measured_peaks()
    bpt = bytes_per_token(w)

    def timed(fn, reps, flush_l2):
        times = []
        for _ in range(reps):
            if flush_l2:
                flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            times.append(e0.elapsed_time(e1))
        return float(np.median(times)), float(np.min(times))

    # calibration: one call over all 262144 tokens, and 128 calls of 2048 continuing one another
    def calib_once():
        k, xk, _ = sr.calibrate(xc, ws=ws)
        sr.build_sign(n, k, xk, d)

    def calib_chunked():
        for i in range(n_cal // 2048):
            k, xk, _ = sr.calibrate(xc[i * 2048:(i + 1) * 2048], ws=ws, accumulate=i > 0, t_offset=i * 2048)
        sr.build_sign(n, k, xk, d)

    calib_once()
    calib_chunked()
    torch.cuda.synchronize(dev)
    cal_bytes = n_cal * n * 2
    one_med, one_min = timed(calib_once, 5, True)
    ch_med, _ = timed(calib_chunked, 3, True)
    k, xk, _ = sr.calibrate(xc, ws=ws)
    del xc
    torch.cuda.synchronize(dev)

    q = torch.empty((Tmax, n // 2), dtype=torch.uint8, device=dev)
    scale = torch.empty(Tmax, dtype=torch.float32, device=dev)
    zero = torch.empty(Tmax, dtype=torch.float32, device=dev)
    rows = []
    sampler = ClockSampler(dev.index)
    with sampler:
        for T in syn.SWEEP_T:
            xs, qs, ss, zs = x[:T], q[:T], scale[:T], zero[:T]

            def call():
                sr.rotate_quant_outlier(xs, d, k, xk, q=qs, scale=ss, zero=zs)

            for _ in range(max(3, args.warmup)):
                call()
            K = 200 if T <= 4096 else max(20, args.steps // 4)
            torch.cuda.synchronize(dev)
            l0 = sr.kernel_launches()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(K):
                call()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            launches = sr.kernel_launches() - l0
            warm_ms = e0.elapsed_time(e1) / K
            cold_ms, _ = timed(call, 20, True)
            graph = graph_replay(torch, call, stream, dev)
            rows.append({"T": T, **graph, "us_per_call_back_to_back": warm_ms * 1e3,
                         "gbs_back_to_back": T * bpt / (warm_ms * 1e-3) / 1e9,
                         "us_per_call_l2_flushed": cold_ms * 1e3,
                         "gbs_l2_flushed": T * bpt / (cold_ms * 1e-3) / 1e9,
                         "tokens_per_s_back_to_back": T / (warm_ms * 1e-3), "steps": K,
                         "gpu_launches": int(launches)})
    top = rows[-1]
    achieved = top["gbs_back_to_back"]
    line = {
        "metric": METRIC, "value": top["tokens_per_s_back_to_back"], "unit": UNIT, "n_gpus": 1,
        "steps": top["steps"], "warmup": max(3, args.warmup), "ms_per_step": top["us_per_call_back_to_back"] * 1e-3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic (8192 drawn rows tiled to 32768; 8192 calibration rows tiled to 262144)",
        "config": {"workload": w.name, "n": n, "sweep_T": list(syn.SWEEP_T), "input_dtype": w.dtype,
                   "quant": "asym4",
                   "l2": "back-to-back rows: inputs below 126 MB stay in L2 (T <= 4096); "
                         "flushed rows: a 252 MB write before each timed call"},
        "sweep": rows,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None, "peak_source": peaks["source"],
                     "bytes_per_token": bpt, "kernel": "signrot_rotate_quant (T = 32768)",
                     "kernel_sources": kernel_sources_digest()},
        "calibration": {
            "tokens": n_cal, "bytes": cal_bytes,
            "one_call_ms": one_med, "one_call_gbs": cal_bytes / (one_med * 1e-3) / 1e9,
            "one_call_frac": cal_bytes / (one_med * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "one_call_ms_min": one_min,
            "chunked_2048_ms": ch_med, "chunked_gbs": cal_bytes / (ch_med * 1e-3) / 1e9,
            "calls": "signrot_calibrate + signrot_build_sign, L2 flushed before each timing"},
        "gpu_launches": top["gpu_launches"],
        "clocks": sampler.report(),
    }
    print(json.dumps(line), flush=True)
    return 0


def main(argv=None) -> int:
    args = parse(argv)
    _default_also(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_sweep(args) if args.sweep else run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
