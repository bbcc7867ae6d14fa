#!/usr/bin/env python
"""AutoRound tuning-step benchmark on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one SignSGD tuning step of a Llama-7B-shaped 4096x4096 linear layer
on 8 samples x 2048 tokens (16384 tokens), W4 asymmetric, group 128, lr 5e-3:
QDQ -> forward GEMM with the MSE residual epilogue -> weight-gradient GEMM with
the straight-through fold and SignSGD update fused in.  Inputs are seeded
synthetic tensors (weights ~N(0, 0.02) with 0.1 % outliers x20, activations
~N(0, 1) with 8 outlier channels x50) standing in for trained weights and
calibration text.

Prints ONE JSON line (rank 0).  ``value`` is tuning steps/s of the whole job
(N ranks each tune their own independent layer: weak scaling, no collective on
the data path).  Extra keys: ``roofline`` (dominant kernel vs the measured bf16
peak), ``cpu_baseline`` (the CPU oracle on a bounded row sample), ``e2e``
(the same metric through the host-buffer API with copies inside the timed
region), ``gpu_launches``, ``clocks``, ``kernels`` (per-kernel device time)
and ``w4a16`` (the INT4 decode matmul on the 8192x28672 down projection).

``--impl reference`` times the CPU oracle itself on the host cores (rank 0
only), on row samples of the same workload.

``--case NAME`` runs one small invocation of one kernel family (three
launches, no timing, no JSON line) for an ncu capture of that kernel; see
``CASES`` below.

Peaks: a kernel's bf16 fraction is taken against the measured burst peak when
its timed region is shorter than a second and against the sustained peak for a
seconds-long loop; both fractions are reported, and the ``sustained`` object
holds the same step loop kept busy for a few seconds.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "AutoRound tuning steps/s per layer (TFLOP/s, % bf16 roofline); W4A16 GEMV % HBM BW"
WORKLOAD = "linear_4096"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SAMPLE_ROWS_CPU = 128
SAMPLE_ROWS_REF = 128


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


SUSTAINED_FROM_S = 1.0  # timed regions shorter than this run at the burst clock


def tensor_peak(peaks, seconds):
    """The bf16 peak that applies to a kernel timed over ``seconds``: the burst
    figure for a short region (the clock has not yet settled under the power
    cap), the sustained one for a seconds-long loop.  Returns (TFLOP/s, label)."""
    burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if seconds < SUSTAINED_FROM_S:
        return burst, f"bf16_tflops (burst): timed region {seconds:.3f} s < {SUSTAINED_FROM_S:g} s"
    return sus, f"bf16_tflops_sustained: timed region {seconds:.2f} s >= {SUSTAINED_FROM_S:g} s"


def both_fracs(peaks, tflops):
    return {"frac_burst": tflops / peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]),
            "frac_sustained": tflops / peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])}


def workload_config(wl, n_gpus):
    return {
        "workload": f"{wl.name}: {wl.n_out}x{wl.n_in} bf16 linear, {wl.m_tokens} tokens (8x2048), "
                    f"W{wl.bits} asym g{wl.group_size}, lr {wl.lr}, one SignSGD step per iteration",
        "n_out": wl.n_out, "n_in": wl.n_in, "tokens": wl.m_tokens, "bits": wl.bits, "group_size": wl.group_size,
        "lr": wl.lr, "layers": n_gpus, "parallelism": f"{n_gpus} independent layers, one per GPU",
        "l2": "inputs larger than L2: X 134 MB and Y 268 MB per layer exceed the 126 MB L2; no flush needed",
    }


# ----------------------------------------------------------------------------
# clocks during the timed region (NVML reads only; nothing is changed)
# ----------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        self._handle = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self._nv = pynvml
            self._handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report what is missing
            self.error = str(e)
        self._thread = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
                for bit, name in self.REASONS.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._handle is not None:
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._handle is not None:
            self._thread.join()

    def summary(self):
        if self._handle is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": getattr(self, "error", "no NVML")}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------------
# traffic of the dominant kernel from the committed ncu summary
# ----------------------------------------------------------------------------

KERNEL_SOURCES = ["post_weight_quantization_autoround_b200/csrc/ar_gemm.cu",
                  "post_weight_quantization_autoround_b200/csrc/ar_device.cuh"]


def gemm_source_hash() -> str:
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel_tag: str):
    """dram bytes per launch recorded in profiles/, or None if missing or the kernel changed since."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}_{WORKLOAD}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_b = re.search(r"dram_bytes_per_launch\s*=\s*([0-9.eE+]+)", text)
    m_h = re.search(r"source_hash\s*=\s*([0-9a-f]+)", text)
    if not m_b or not m_h or m_h.group(1) != gemm_source_hash():
        return None
    return float(m_b.group(1))


# ----------------------------------------------------------------------------
# the CPU oracle on a bounded sample (rank 0, N = 1) and the reference arm
# ----------------------------------------------------------------------------

def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        return max(i.get("num_threads", 1) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


class OracleSample:
    """The oracle's tuning step on ``rows`` of the layer's output rows (rows are independent)."""

    def __init__(self, wl, d, rows):
        from oracle import autoround_oracle as O

        self.O = O
        self.wl = wl
        idx = np.arange(rows)
        self.W = synth.bf16_bits_to_f32(d["W"][idx])
        self.X = synth.bf16_bits_to_f32(d["X"])
        self.Y = O.reference_forward(self.X, self.W)
        self.V, self.a, self.b = synth.make_state(rows, wl.n_in, wl.group_size)
        self.cfg = O.QConfig(bits=wl.bits, group_size=wl.group_size, lr=wl.lr)
        self.count = wl.m_tokens * wl.n_out
        self.scale = wl.n_out / rows  # sample -> whole layer

    def step(self):
        _, (self.V, self.a, self.b), _, _ = self.O.tune_step_linear(self.W, self.X, self.Y, self.V, self.a, self.b,
                                                                    self.cfg, count=self.count)


def cpu_baseline(wl, d, budget_s=10.0):
    """The oracle on a bounded row sample, on one host thread (the plain baseline) and on all BLAS threads."""
    from threadpoolctl import threadpool_limits

    s = OracleSample(wl, d, SAMPLE_ROWS_CPU)
    out = {}
    for label, limit in (("single", 1), ("multi", None)):
        with threadpool_limits(limits=limit):
            cores = blas_threads()
            s.step()  # warm
            n, t0 = 0, time.perf_counter()
            while True:
                s.step()
                n += 1
                el = time.perf_counter() - t0
                if el >= budget_s / 2:
                    break
        per_layer_step = el / n * s.scale
        out[label] = {"value": 1.0 / per_layer_step, "unit": "steps/s", "cores": cores, "kind": "oracle",
                      "extrapolated": True,
                      "sample": f"{n} oracle steps on {SAMPLE_ROWS_CPU} of {wl.n_out} output rows (rows are "
                                f"independent), {el:.1f} s, time scaled x{s.scale:g} to the full layer"}
    res = dict(out["single"])
    res["multi_thread"] = out["multi"]
    return res


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    d = synth.make_linear(wl.n_out, wl.n_in, wl.m_tokens, seed=wl.seed)
    s = OracleSample(wl, d, SAMPLE_ROWS_REF)
    for _ in range(args.warmup):
        s.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        s.step()
    el = time.perf_counter() - t0
    value = args.steps / (el * s.scale)
    sample = (f"each step: the oracle's SignSGD step on {SAMPLE_ROWS_REF} of {wl.n_out} output rows "
              f"(exact, rows are independent); value extrapolated: time scaled x{s.scale:g} to the full layer")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, 1),
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": blas_threads(), "kind": "oracle",
                         "extrapolated": True, "sample": sample},
        "timed_s": el, "extrapolated": f"x{s.scale:g} from a {SAMPLE_ROWS_REF}-row sample",
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def to_dev_bf16(bits, torch):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def w4a16_bench(ar, torch, peaks, reps=20):
    wl = synth.WORKLOADS["down_8192_28672"]
    N, K, g = wl.n_out, wl.n_in, wl.group_size
    d = synth.make_linear(N, K, 1, seed=wl.seed, x_outlier_channels=0)
    Wd = to_dev_bf16(d["W"], torch)
    V = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    a = torch.ones((N, K // g), dtype=torch.float32, device="cuda")
    b = torch.ones((N, K // g), dtype=torch.float32, device="cuda")
    cfg = ar.ar_qconfig_default(bits=4, group_size=g)
    packed = torch.empty((N, K // 8), dtype=torch.int32, device="cuda")
    s16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    z16 = torch.empty((N, K // g), dtype=torch.float16, device="cuda")
    ar.ar_pack_int4(Wd, V, a, b, cfg, packed, s16, z16)
    del Wd, V
    # L2 flush by reading 256 MB (a write would leave dirty lines whose write-back
    # competes with the measured kernel)
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.int32, device="cuda")
    out = {}
    for T in (1, 4, 16, 256):
        A = to_dev_bf16(synth.make_activations(T, K, seed=T), torch)
        y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            ar.ar_w4a16_gemm(A, packed, s16, z16, g, y)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in ev:
            flush.sum()  # evict the 117 MB of packed weights from L2
            e0.record()
            ar.ar_w4a16_gemm(A, packed, s16, z16, g, y)
            e1.record()
        torch.cuda.synchronize()
        ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
        nbytes = packed.numel() * 4 + s16.numel() * 2 + z16.numel() * 2 + A.numel() * 2 + y.numel() * 2
        gbs = nbytes / (ms * 1e-3) / 1e9
        flops = 2.0 * T * N * K
        tfs = flops / (ms * 1e-3) / 1e12
        peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        # roofline: the slower of the HBM time of the bytes and the tensor time of the FLOPs
        t_roof = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (peak_tf * 1e12))
        out[f"T{T}"] = {"us": ms * 1e3, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"], "TFLOP/s": tfs,
                        "bound": "hbm" if nbytes / peaks["hbm_gbs"] / 1e9 >= flops / peak_tf / 1e12 else "tensor",
                        "roofline_frac": t_roof / (ms * 1e-3),
                        "algorithmic_bytes": nbytes, "kernel": ar.ar_last_kernels()}
    out["shape"] = f"{N}x{K} int4 g{g}, fp16 scale/zero, bf16 activations; L2 flushed before each launch"
    # the same layer packed at 2, 3 and 8 bits (T = 1: the decode kernel at 2 and 3 bits, the tcgen05
    # dequant GEMM at 8 bits; T = 256: the tcgen05 dequant GEMM)
    W = to_dev_bf16(d["W"], torch)
    V = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    for bits in (2, 3, 8):
        cfgb = ar.ar_qconfig_default(bits=bits, group_size=g)
        pk = torch.empty((N, K * bits // 32), dtype=torch.int32, device="cuda")
        ar.ar_pack_codes(W, V, a, b, cfgb, pk, s16, z16)
        for T in (1, 256):
            A = to_dev_bf16(synth.make_activations(T, K, seed=T), torch)
            y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
            for _ in range(3):
                ar.ar_wxa16_gemm(A, pk, s16, z16, g, bits, y)
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            for e0, e1 in ev:
                flush.sum()
                e0.record()
                ar.ar_wxa16_gemm(A, pk, s16, z16, g, bits, y)
                e1.record()
            torch.cuda.synchronize()
            ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
            nbytes = pk.numel() * 4 + s16.numel() * 2 + z16.numel() * 2 + A.numel() * 2 + y.numel() * 2
            out[f"W{bits}A16_T{T}"] = {"us": ms * 1e3, "GB/s": nbytes / (ms * 1e-3) / 1e9, "algorithmic_bytes": nbytes,
                                      "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                      "TFLOP/s": 2.0 * T * N * K / (ms * 1e-3) / 1e12, "kernel": ar.ar_last_kernels()}
    # the same layer exported as NVFP4 (E2M1 codes, E4M3 scale per 16 values, per-tensor scale) through
    # the tcgen05 dequant GEMM: 0.5 B per weight + 1 B per 16 weights
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    gs = torch.empty(1, dtype=torch.float32, device="cuda")
    codes = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
    ar.ar_absmax_bf16(W, amax)
    ar.ar_qdq_nvfp4(W, None, None, amax, None, codes, scales, gs)
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    for T in (1, 16, 256):
        A = to_dev_bf16(synth.make_activations(T, K, seed=T), torch)
        y = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
        for _ in range(3):
            ar.ar_nvfp4_gemm(A, codes, scales, gs, y)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for e0, e1 in ev:
            flush.sum()
            e0.record()
            ar.ar_nvfp4_gemm(A, codes, scales, gs, y)
            e1.record()
        torch.cuda.synchronize()
        ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
        nbytes = codes.numel() + scales.numel() + A.numel() * 2 + y.numel() * 2
        flops = 2.0 * T * N * K
        out[f"NVFP4A16_T{T}"] = {"us": ms * 1e3, "GB/s": nbytes / (ms * 1e-3) / 1e9, "algorithmic_bytes": nbytes,
                                 "frac_hbm": nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                 "TFLOP/s": flops / (ms * 1e-3) / 1e12,
                                 "frac_bf16_burst": flops / (ms * 1e-3) / 1e12 / peak_tf,
                                 "kernel": ar.ar_last_kernels()}
    del W, V, codes, scales
    return out


def nvfp4_bench(ar, torch, peaks, reps=20):
    """NVFP4 QDQ (E2M1 codes, E4M3 scale per 16 values, per-tensor scale) of the 4096² and 8192x28672
    layers with offsets V and clip factors alpha; outputs Ŵ, packed codes and scale codes.  L2 flushed
    before each launch.  HBM bytes per weight: W 2 + V 4 + Ŵ 2 + codes 0.5, plus 4 + 1 per 16 (alpha,
    scale code); the absmax pass reads W once more (2 B per weight)."""
    out = {}
    flush = torch.ones(64 * 1024 * 1024, dtype=torch.int32, device="cuda")
    for name, (N, K) in (("linear_4096", (4096, 4096)), ("down_8192_28672", (8192, 28672))):
        d = synth.make_linear(N, K, 1, seed=3, x_outlier_channels=0)
        W = to_dev_bf16(d["W"], torch)
        del d
        V = (torch.rand((N, K), device="cuda") - 0.5).float()
        a = (torch.rand((N, K // 16), device="cuda") * 0.5 + 0.5).float()
        amax = torch.empty(1, dtype=torch.float32, device="cuda")
        gs = torch.empty(1, dtype=torch.float32, device="cuda")
        What = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        codes = torch.empty((N, K // 2), dtype=torch.uint8, device="cuda")
        scales = torch.empty((N, K // 16), dtype=torch.uint8, device="cuda")
        ar.ar_absmax_bf16(W, amax)
        for _ in range(3):
            ar.ar_qdq_nvfp4(W, V, a, amax, What, codes, scales, gs)
        res, kern = {}, {}
        for what, fn in (("qdq", lambda: ar.ar_qdq_nvfp4(W, V, a, amax, What, codes, scales, gs)),
                         ("absmax", lambda: ar.ar_absmax_bf16(W, amax))):
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
            for e0, e1 in ev:
                flush.sum()
                e0.record()
                fn()
                e1.record()
            torch.cuda.synchronize()
            res[what] = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
            kern[what] = ar.ar_last_kernels()
        n = N * K
        qbytes = n * (2 + 4 + 2 + 0.5) + (n // 16) * (4 + 1)
        out[name] = {"qdq_us": res["qdq"] * 1e3, "qdq_GB/s": qbytes / (res["qdq"] * 1e-3) / 1e9,
                     "qdq_frac_hbm": qbytes / (res["qdq"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "absmax_us": res["absmax"] * 1e3,
                     "absmax_frac_hbm": 2.0 * n / (res["absmax"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                     "algorithmic_bytes": qbytes, "kernels": kern}
        del W, V, a, What, codes, scales
    out["format"] = "NVFP4: E2M1 codes, E4M3 scale per 16 values, fp32 tensor scale amax/2688; V and alpha applied"
    # tuning steps on NVFP4 on the 4096² layer with 16384 tokens (the integer step's workload)
    wl = synth.WORKLOADS[WORKLOAD]
    N, K, M = wl.n_out, wl.n_in, wl.m_tokens
    d = synth.make_linear(N, K, M, seed=wl.seed)
    W, X = to_dev_bf16(d["W"], torch), to_dev_bf16(d["X"], torch)
    del d
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ar.ar_linear_forward(X, W, Y)
    V = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    a = torch.ones((N, K // 16), dtype=torch.float32, device="cuda")
    amax = torch.empty(1, dtype=torch.float32, device="cuda")
    ar.ar_absmax_bf16(W, amax)
    steps = 20
    ws = torch.empty(ar.ar_tune_step_nvfp4_workspace(M, N, K, steps), dtype=torch.uint8, device="cuda")
    loss = torch.empty(steps, dtype=torch.float32, device="cuda")
    cfg = ar.ar_qconfig_default()
    ar.ar_tune_step_nvfp4(W, V, a, amax, X, Y, cfg, 3, loss, ws)  # warm-up
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    ar.ar_tune_step_nvfp4(W, V, a, amax, X, Y, cfg, steps, loss, ws)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    flops = 4.0 * M * N * K
    tfs = flops / (ms * 1e-3) / 1e12
    peak, plabel = tensor_peak(peaks, ms * steps * 1e-3)
    lv = loss.cpu().numpy()
    out["tune_linear_4096"] = {"steps_per_s": 1e3 / ms, "ms_per_step": ms, "tflops": tfs, "frac": tfs / peak,
                               "peak": plabel, **both_fracs(peaks, tfs),
                               "steps": steps, "first_loss": float(lv[0]), "last_loss": float(lv[-1]),
                               "kernels": ar.ar_last_kernels()}
    del W, X, Y, V, a, ws
    return out


# ----------------------------------------------------------------------------
# multi-rank plumbing (independent layers per rank; timing only crosses ranks)
# ----------------------------------------------------------------------------

def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank tunes its own independent layer."""
    return base_seed + rank


def max_over_ranks(value: float, dist, device) -> float:
    """Largest value over all ranks (the job's device time); identity without a process group."""
    import torch

    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps: int, max_ms: float) -> float:
    """Whole-job steps/s: every rank ran `steps` steps; the job took the slowest rank's time."""
    return world * steps / (max_ms * 1e-3)


_LAST_PROFILE = {}


def _time_call(torch, fn, warmup=1, ar=None):
    """Device time (ms) of one call of fn; with ``ar`` the per-kernel device times of that call are kept in
    _LAST_PROFILE (the library's event profiler; it adds two events per launch)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    _LAST_PROFILE.clear()
    if ar is not None:
        ar.ar_profile_start()
        fn()
        torch.cuda.synchronize()
        _LAST_PROFILE.update(ar.ar_profile_stop())
    return ms


def _kernel_split(n_steps):
    """Per-kernel share of the last profiled call: {name: [launches, us per step]}."""
    return {k: [n, round(1e3 * t / n_steps, 2)] for k, (n, t) in sorted(_LAST_PROFILE.items(), key=lambda kv: -kv[1][1])}


def other_workloads(ar, torch, peaks, steps=10):
    """Tuning throughput on the remaining workloads (one call of ``steps`` steps each)."""
    out = {}

    def fracs(tfs, seconds):
        peak, label = tensor_peak(peaks, seconds)
        return {"frac": tfs / peak, "peak": label, **both_fracs(peaks, tfs)}

    # SwiGLU MLP block, tuned jointly
    wl = synth.WORKLOADS["mlp_4096_11008"]
    M, Hd, F = wl.m_tokens, wl.n_in, wl.inter
    d = synth.make_mlp(Hd, F, M, seed=wl.seed)
    Ws = [to_dev_bf16(d[k], torch) for k in ("Wg", "Wu", "Wd")]
    X = to_dev_bf16(d["X"], torch)
    del d
    g = wl.group_size
    st = [(torch.zeros(W.shape, device="cuda"), torch.ones((W.shape[0], W.shape[1] // g), device="cuda"),
           torch.ones((W.shape[0], W.shape[1] // g), device="cuda")) for W in Ws]
    cfg = ar.ar_qconfig_default(bits=wl.bits, group_size=g, lr=wl.lr)
    Y = torch.empty((M, Hd), device="cuda")
    fws = torch.empty(ar.ar_block_forward_workspace(ar.AR_BLOCK_SWIGLU_MLP, Ws, M), dtype=torch.uint8, device="cuda")
    ar.ar_block_forward(ar.AR_BLOCK_SWIGLU_MLP, Ws, X, Y, fws)
    del fws
    layers = [(W, *s) for W, s in zip(Ws, st)]
    ws = torch.empty(ar.ar_tune_block_workspace(ar.AR_BLOCK_SWIGLU_MLP, layers, M, cfg, steps), dtype=torch.uint8,
                     device="cuda")
    loss = torch.empty(steps, device="cuda")
    ms = _time_call(torch, lambda: ar.ar_tune_block(ar.AR_BLOCK_SWIGLU_MLP, layers, X, Y, cfg, steps, loss, ws))
    flops = 14.0 * M * Hd * F
    out[wl.name] = {"steps_per_s": steps / (ms * 1e-3), "ms_per_step": ms / steps,
                    "tflops": flops * steps / (ms * 1e-3) / 1e12,
                    **fracs(flops * steps / (ms * 1e-3) / 1e12, ms * 1e-3),
                    "kernels": ar.ar_last_kernels().count(";") + 1, "steps": steps,
                    "final_loss": float(loss[-1].item())}
    del Ws, X, Y, st, layers, ws
    torch.cuda.empty_cache()
    # single linear layers: low-bit stress and the 70B-shaped down projection
    for name in ("lowbit_b3g32", "lowbit_b2g32", "lowbit_b8g256", "down_8192_28672"):
        wl = synth.WORKLOADS[name]
        N, K, M, g = wl.n_out, wl.n_in, wl.m_tokens, wl.group_size
        d = synth.make_linear(N, K, M, seed=wl.seed)
        W, X = to_dev_bf16(d["W"], torch), to_dev_bf16(d["X"], torch)
        del d
        V = torch.zeros((N, K), device="cuda")
        a = torch.ones((N, K // g), device="cuda")
        b = torch.ones((N, K // g), device="cuda")
        cfg = ar.ar_qconfig_default(bits=wl.bits, group_size=g, lr=wl.lr)
        Y = torch.empty((M, N), device="cuda")
        ar.ar_linear_forward(X, W, Y)
        n = steps if name.startswith("down") else 5 * steps
        ws = torch.empty(ar.ar_tune_step_workspace(W, V, a, b, M, cfg, n), dtype=torch.uint8, device="cuda")
        loss = torch.empty(n, device="cuda")
        ms = _time_call(torch, lambda: ar.ar_tune_step(W, V, a, b, X, Y, cfg, n, loss, ws), ar=ar)
        flops = 4.0 * M * N * K
        out[name] = {"steps_per_s": n / (ms * 1e-3), "ms_per_step": ms / n, "tflops": flops * n / (ms * 1e-3) / 1e12,
                     **fracs(flops * n / (ms * 1e-3) / 1e12, ms * 1e-3), "steps": n,
                     "kernels_us_per_step": _kernel_split(n),
                     "final_loss": float(loss[-1].item())}
        del W, X, V, a, b, Y, ws
        torch.cuda.empty_cache()
    # the decoder block (attention + MLP, seven tuned weights) at the Llama-7B shapes, 8 x 2048 tokens
    steps_d = 5
    fn, flops_d, loss_d = decoder_step_fn(ar, torch, 8, 2048, steps_d)
    ms = _time_call(torch, fn, ar=ar)
    out["decoder_llama7b_16384"] = {
        "kernels_us_per_step": _kernel_split(steps_d),
        "steps_per_s": steps_d / (ms * 1e-3), "ms_per_step": ms / steps_d,
        "tflops": flops_d * steps_d / (ms * 1e-3) / 1e12, **fracs(flops_d * steps_d / (ms * 1e-3) / 1e12, ms * 1e-3),
        "steps": steps_d, "first_loss": float(loss_d[0].item()), "last_loss": float(loss_d[-1].item()),
        "kernels": ar.ar_last_kernels().count(";") + 1,
        "note": "H 4096, F 11008, 32 heads of 128, 8 samples x 2048 tokens, W4 g128; FLOPs: the seven tuned GEMMs "
                "(x3 for forward and backward) plus causal attention's six products"}
    del fn, loss_d
    torch.cuda.empty_cache()
    # block-by-block tuning of two SwiGLU blocks with the "light" preset: every step of the
    # method (reference forwards over all samples, gathered minibatch steps, quantized forwards)
    from post_weight_quantization_autoround_b200 import driver

    pre = driver.PRESETS["light"]
    Hd, F = 4096, 11008
    S, Lq, Bq, iters = pre["samples"], pre["seqlen"], pre["batch"], pre["iters"]
    raw = [synth.make_mlp(Hd, F, 1, seed=40 + b) for b in range(2)]
    blocks = [[to_dev_bf16(d[k], torch) for k in ("Wg", "Wu", "Wd")] for d in raw]
    del raw
    X0 = to_dev_bf16(synth.make_activations(S * Lq, Hd, seed=41), torch).view(S, Lq, Hd)
    sched = synth.make_schedule(S, Bq, iters, seed=0)
    cfg = ar.ar_qconfig_default(bits=4, group_size=128, lr=driver.LR)
    driver.tune_mlp_blocks(blocks[:1], X0, cfg, sched[:2])  # allocations and first launches
    ms = _time_call(torch, lambda: driver.tune_mlp_blocks(blocks, X0, cfg, sched), warmup=0)
    flops = 2 * (2 * 6.0 * S * Lq * Hd * F + iters * 14.0 * Bq * Lq * Hd * F)
    out["driver_light_2x_mlp_4096_11008"] = {
        "blocks": 2, "preset": "light", "samples": S, "seqlen": Lq, "batch": Bq, "iters": iters,
        "s_per_block": ms / 2e3, "steps_per_s": 2 * iters / (ms * 1e-3),
        "tflops": flops / (ms * 1e-3) / 1e12, **fracs(flops / (ms * 1e-3) / 1e12, ms * 1e-3),
        "note": "per block: reference forward on all samples, 50 gathered-minibatch joint steps, quantized forward"}
    del blocks, X0
    torch.cuda.empty_cache()
    if ar.ar_get_device_status() != 0:
        out["device_status"] = ar.ar_last_error()
    return out


# ----------------------------------------------------------------------------
# single-kernel cases for ncu captures (inputs larger than L2, a few GB at most)
# ----------------------------------------------------------------------------

def decoder_step_fn(ar, torch, samples, seqlen, steps, H=4096, F=11008, nh=32, g=128):
    """A Llama-7B-shaped decoder block (H 4096, F 11008, 32 heads) on ``samples`` x ``seqlen`` tokens: returns
    (a call running ``steps`` joint tuning steps, FLOPs per step).  Synthetic weights and activations."""
    M = samples * seqlen
    d = synth.make_decoder(H, F, M, seed=7)
    names = ar.DECODER_LAYERS
    Ws = [to_dev_bf16(d[n], torch) for n in names]
    X = to_dev_bf16(d["X"], torch)
    g1 = torch.from_numpy(d["gamma1"]).cuda()
    g2 = torch.from_numpy(d["gamma2"]).cuda()
    del d
    layers = [(W, torch.zeros(W.shape, device="cuda"), torch.ones((W.shape[0], W.shape[1] // g), device="cuda"),
               torch.ones((W.shape[0], W.shape[1] // g), device="cuda")) for W in Ws]
    Y = torch.empty((M, H), device="cuda")
    fws = torch.empty(ar.ar_decoder_forward_workspace(H, F, nh, seqlen, M), dtype=torch.uint8, device="cuda")
    ar.ar_decoder_forward(Ws, g1, g2, nh, seqlen, X, Y, fws)
    del fws
    cfg = ar.ar_qconfig_default(group_size=g)
    ws = torch.empty(ar.ar_tune_step_decoder_workspace(layers, g1, g2, nh, seqlen, M, cfg, steps), dtype=torch.uint8,
                     device="cuda")
    loss = torch.empty(steps, device="cuda")
    fn = lambda: ar.ar_tune_step_decoder(layers, g1, g2, nh, seqlen, X, Y, cfg, steps, loss, ws)
    # the seven tuned GEMMs, forward and backward (2 MNK each, x3), plus causal attention
    # (Q K^T and P V forward; dO V^T, P^T dO, dS K, dS^T Q backward; half the keys each; the scores the
    # two-pass softmax and the backward recompute are not counted)
    gemm = 2.0 * M * (4 * H * H + 3 * H * F) * 3
    attn = 2.0 * samples * nh * seqlen * seqlen * (H // nh) * 6 / 2
    return fn, gemm + attn, loss


def run_case(name, ar, torch):
    """Three launches of one kernel family on a small case (for ``ncu -k <kernel> -s 2 -c 1``)."""
    dev = "cuda"
    if name in ("qdq", "pack_int4", "qdq_nvfp4", "absmax"):
        N, K, g = 8192, 8192, 128  # W 134 MB + V 268 MB: beyond the 126 MB L2
        d = synth.make_linear(N, K, 1, seed=5, x_outlier_channels=0)
        W = to_dev_bf16(d["W"], torch)
        V = (torch.rand((N, K), device=dev) - 0.5).float()
        if name in ("qdq", "pack_int4"):
            a = (torch.rand((N, K // g), device=dev) * 0.5 + 0.5).float()
            b = (torch.rand((N, K // g), device=dev) * 0.5 + 0.5).float()
            cfg = ar.ar_qconfig_default(bits=4, group_size=g)
            if name == "qdq":  # as in the tuning step: W_hat, scale, zero
                What = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
                sc = torch.empty((N, K // g), device=dev)
                zp = torch.empty((N, K // g), device=dev)
                fn = lambda: ar.ar_qdq(W, V, a, b, cfg, What, None, sc, zp)
            else:
                pk = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
                s16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
                z16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
                fn = lambda: ar.ar_pack_int4(W, V, a, b, cfg, pk, s16, z16)
        else:
            a = (torch.rand((N, K // 16), device=dev) * 0.5 + 0.5).float()
            amax = torch.empty(1, device=dev)
            ar.ar_absmax_bf16(W, amax)
            if name == "absmax":
                fn = lambda: ar.ar_absmax_bf16(W, amax)
            else:
                What = torch.empty((N, K), dtype=torch.bfloat16, device=dev)
                codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
                scales = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
                gs = torch.empty(1, device=dev)
                fn = lambda: ar.ar_qdq_nvfp4(W, V, a, amax, What, codes, scales, gs)
    elif name == "tune_nvfp4":  # one NVFP4 tuning step per launch set: qdq_nvfp4, GEMMs, fold_nvfp4
        N, K, M = 4096, 4096, 4096
        d = synth.make_linear(N, K, M, seed=5)
        W, X = to_dev_bf16(d["W"], torch), to_dev_bf16(d["X"], torch)
        Y = torch.empty((M, N), device=dev)
        ar.ar_linear_forward(X, W, Y)
        V = torch.zeros((N, K), device=dev)
        a = torch.ones((N, K // 16), device=dev)
        amax = torch.empty(1, device=dev)
        ar.ar_absmax_bf16(W, amax)
        ws = torch.empty(ar.ar_tune_step_nvfp4_workspace(M, N, K, 1), dtype=torch.uint8, device=dev)
        loss = torch.empty(1, device=dev)
        cfg = ar.ar_qconfig_default()
        fn = lambda: ar.ar_tune_step_nvfp4(W, V, a, amax, X, Y, cfg, 1, loss, ws)
    elif name == "mlp":  # one joint SwiGLU step: swiglu_fwd, resid, fold x3, swiglu_bwd GEMMs
        Hd, F, M = 4096, 11008, 2048
        d = synth.make_mlp(Hd, F, M, seed=5)
        Ws = [to_dev_bf16(d[k], torch) for k in ("Wg", "Wu", "Wd")]
        X = to_dev_bf16(d["X"], torch)
        st = [(torch.zeros(W.shape, device=dev), torch.ones((W.shape[0], W.shape[1] // 128), device=dev),
               torch.ones((W.shape[0], W.shape[1] // 128), device=dev)) for W in Ws]
        Y = torch.empty((M, Hd), device=dev)
        fws = torch.empty(ar.ar_block_forward_workspace(ar.AR_BLOCK_SWIGLU_MLP, Ws, M), dtype=torch.uint8, device=dev)
        ar.ar_block_forward(ar.AR_BLOCK_SWIGLU_MLP, Ws, X, Y, fws)
        layers = [(W, *t) for W, t in zip(Ws, st)]
        cfg = ar.ar_qconfig_default()
        ws = torch.empty(ar.ar_tune_block_workspace(ar.AR_BLOCK_SWIGLU_MLP, layers, M, cfg, 1), dtype=torch.uint8,
                         device=dev)
        loss = torch.empty(1, device=dev)
        fn = lambda: ar.ar_tune_block(ar.AR_BLOCK_SWIGLU_MLP, layers, X, Y, cfg, 1, loss, ws)
    elif name == "decoder":  # one joint step of a Llama-7B-shaped decoder block on one 2048-token sample
        fn = decoder_step_fn(ar, torch, 1, 2048, 1)[0]
    elif name == "lowbit_b2g32":  # two tuning steps per call of the W2 g32 4096 x 4096 layer, 2048 tokens
        wl = synth.WORKLOADS[name]
        N, K, M, g = wl.n_out, wl.n_in, wl.m_tokens, wl.group_size
        d = synth.make_linear(N, K, M, seed=wl.seed)
        W, X = to_dev_bf16(d["W"], torch), to_dev_bf16(d["X"], torch)
        del d
        V = torch.zeros((N, K), device=dev)
        a = torch.ones((N, K // g), device=dev)
        b = torch.ones((N, K // g), device=dev)
        cfg = ar.ar_qconfig_default(bits=wl.bits, group_size=g, lr=wl.lr)
        Y = torch.empty((M, N), device=dev)
        ar.ar_linear_forward(X, W, Y)
        ws = torch.empty(ar.ar_tune_step_workspace(W, V, a, b, M, cfg, 2), dtype=torch.uint8, device=dev)
        loss = torch.empty(2, device=dev)
        fn = lambda: ar.ar_tune_step(W, V, a, b, X, Y, cfg, 2, loss, ws)
    elif name in ("w4a16_t1", "w2a16_t1", "w8a16_t1", "w3a16_t256", "nvfp4_gemm_t1", "nvfp4_gemm_t256"):  # the 8192 x 28672 layer's exports
        N, K, g = 8192, 28672, 128
        d = synth.make_linear(N, K, 1, seed=5, x_outlier_channels=0)
        W = to_dev_bf16(d["W"], torch)
        del d
        T = 256 if name.endswith("t256") else 1
        A = to_dev_bf16(synth.make_activations(T, K, seed=T), torch)
        y = torch.empty((T, N), dtype=torch.bfloat16, device=dev)
        if name in ("w3a16_t256", "w2a16_t1", "w8a16_t1"):
            bits = {"w3a16_t256": 3, "w2a16_t1": 2, "w8a16_t1": 8}[name]
            V = torch.zeros((N, K), device=dev)
            a = torch.ones((N, K // g), device=dev)
            pk = torch.empty((N, K * bits // 32), dtype=torch.int32, device=dev)
            s16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
            z16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
            ar.ar_pack_codes(W, V, a, a, ar.ar_qconfig_default(bits=bits, group_size=g), pk, s16, z16)
            del V, a
            fn = lambda: ar.ar_wxa16_gemm(A, pk, s16, z16, g, bits, y)
        elif name == "w4a16_t1":
            V = torch.zeros((N, K), device=dev)
            a = torch.ones((N, K // g), device=dev)
            pk = torch.empty((N, K // 8), dtype=torch.int32, device=dev)
            s16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
            z16 = torch.empty((N, K // g), dtype=torch.float16, device=dev)
            ar.ar_pack_int4(W, V, a, a, ar.ar_qconfig_default(bits=4, group_size=g), pk, s16, z16)
            del V, a
            fn = lambda: ar.ar_w4a16_gemm(A, pk, s16, z16, g, y)
        else:
            amax = torch.empty(1, device=dev)
            gs = torch.empty(1, device=dev)
            codes = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
            scales = torch.empty((N, K // 16), dtype=torch.uint8, device=dev)
            ar.ar_absmax_bf16(W, amax)
            ar.ar_qdq_nvfp4(W, None, None, amax, None, codes, scales, gs)
            fn = lambda: ar.ar_nvfp4_gemm(A, codes, scales, gs, y)
        del W
        torch.cuda.synchronize()
        torch.cuda.empty_cache()  # only the exports, activations and output stay on the device
    else:
        raise SystemExit(f"unknown case {name}; one of {', '.join(CASES)}")
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    st = ar.ar_get_device_status()
    print(f"case {name}: kernels {ar.ar_last_kernels()} status {st}", flush=True)
    return 0 if st == 0 else 1


CASES = ("qdq", "pack_int4", "qdq_nvfp4", "absmax", "tune_nvfp4", "mlp", "decoder", "lowbit_b2g32", "w4a16_t1",
         "w2a16_t1", "w8a16_t1", "w3a16_t256", "nvfp4_gemm_t1", "nvfp4_gemm_t256")


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-w4a16", action="store_true")
    ap.add_argument("--no-nvfp4", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other workloads (MLP, low-bit, 70B down)")
    ap.add_argument("--no-sustained", action="store_true", help="skip the seconds-long sustained loop")
    ap.add_argument("--case", choices=CASES, help="run one small kernel case for an ncu capture and exit")
    ap.add_argument("--sustained-s", type=float, default=3.0, help="length of the sustained loop (wall seconds)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = synth.WORKLOADS[WORKLOAD]
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch
    import torch.distributed as dist

    import post_weight_quantization_autoround_b200 as ar

    if args.case:
        return run_case(args.case, ar, torch)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    peaks, peaks_src = load_peaks()

    # --- inputs: each rank tunes its own independent layer
    d = synth.make_linear(wl.n_out, wl.n_in, wl.m_tokens, seed=rank_seed(wl.seed, rank))
    cfg = ar.ar_qconfig_default(bits=wl.bits, group_size=wl.group_size, lr=wl.lr)
    W = to_dev_bf16(d["W"], torch)
    X = to_dev_bf16(d["X"], torch)
    N, K, M, g = wl.n_out, wl.n_in, wl.m_tokens, wl.group_size
    V = torch.zeros((N, K), dtype=torch.float32, device="cuda")
    alpha = torch.ones((N, K // g), dtype=torch.float32, device="cuda")
    beta = torch.ones((N, K // g), dtype=torch.float32, device="cuda")
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ar.ar_linear_forward(X, W, Y)
    n_max = max(args.steps, args.warmup, 200)
    ws = torch.empty(ar.ar_tune_step_workspace(W, V, alpha, beta, M, cfg, n_max), dtype=torch.uint8, device="cuda")
    loss = torch.empty(n_max, dtype=torch.float32, device="cuda")

    def steps(n):
        # one call runs n tuning steps (QDQ, forward GEMM, weight-gradient GEMM each)
        ar.ar_tune_step(W, V, alpha, beta, X, Y, cfg, n, loss, ws)

    steps(args.warmup)
    torch.cuda.synchronize()
    if ar.ar_get_device_status() != 0:
        raise SystemExit(f"device status after warm-up: {ar.ar_last_error()}")

    # --- timed region: exactly K steps, barrier + synchronize on both sides
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        ar.ar_profile_start()
        e0.record(stream)
        steps(args.steps)
        e1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        prof = ar.ar_profile_stop()
    ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, "cuda")
    status = ar.ar_get_device_status()
    final_loss = float(loss[args.steps - 1].item())

    launches = sum(n for n, _ in prof.values())
    kernels = {k: {"launches": n, "ms_total": t_ms, "us_per_launch": 1e3 * t_ms / max(n, 1),
                   "share": t_ms / max(sum(x[1] for x in prof.values()), 1e-12)} for k, (n, t_ms) in prof.items()}
    flops_gemm = 2.0 * M * N * K
    flops_step = 2 * flops_gemm
    steps_s_rank = args.steps / (ms * 1e-3)
    value = job_throughput(world, args.steps, ms)
    gemm_names = [k for k in prof if k.startswith("umma_gemm")]
    dom = max(gemm_names, key=lambda k: prof[k][1])
    dom_us = kernels[dom]["us_per_launch"]
    achieved = flops_gemm / (dom_us * 1e-6) / 1e12
    # the peak that applies to this timed region: burst for a short one, sustained for a seconds-long one
    peak, peak_label = tensor_peak(peaks, ms * 1e-3)
    tag = "fwd_gemm" if "resid" in dom else "wgrad_fold_gemm"
    traffic = profiled_traffic(tag)
    step_tflops = flops_step * steps_s_rank / 1e12
    result = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; Llama-7B-shaped layer and calibration stand-ins)",
        "config": workload_config(wl, world),
        "tflops": step_tflops * world,
        "step_roofline_frac": step_tflops / peak,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, **both_fracs(peaks, achieved),
                     "peak_source": f"{peaks_src} {peak_label}",
                     "algorithmic_flops_per_launch": flops_gemm},
        "gpu_launches": launches,
        "kernels": kernels,
        "clocks": clocks.summary(),
        "device_status": status,
        "final_loss": final_loss,
    }

    # --- the same step loop held for seconds (the clock settles under the power cap): sustained figures
    if not args.no_sustained:
        calls, chunk = 0, min(n_max, 200)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(local) as sclk:
            torch.cuda.synchronize()
            ar.ar_profile_start()
            s0.record(stream)
            t_wall = time.perf_counter()
            while time.perf_counter() - t_wall < args.sustained_s:
                steps(chunk)
                calls += 1
                if calls % 4 == 0:
                    torch.cuda.synchronize()
            s1.record(stream)
            torch.cuda.synchronize()
            sprof = ar.ar_profile_stop()
        sms = s0.elapsed_time(s1)
        n_sus = calls * chunk
        sdom_us = 1e3 * sprof[dom][1] / max(sprof[dom][0], 1)
        sach = flops_gemm / (sdom_us * 1e-6) / 1e12
        speak, slabel = tensor_peak(peaks, sms * 1e-3)
        result["sustained"] = {
            "steps": n_sus, "seconds": sms * 1e-3, "steps_per_s": n_sus / (sms * 1e-3),
            "ms_per_step": sms / n_sus, "tflops": flops_step * n_sus / (sms * 1e-3) / 1e12,
            "step_roofline_frac": flops_step * n_sus / (sms * 1e-3) / 1e12 / speak,
            "kernel": dom, "kernel_us_per_launch": sdom_us, "kernel_tflops": sach, "kernel_frac": sach / speak,
            **{f"kernel_{k}": v for k, v in both_fracs(peaks, sach).items()},
            "peak_source": f"{peaks_src} {slabel}", "clocks": sclk.summary(),
            "note": f"{calls} back-to-back calls of {chunk} steps; device time over the whole loop"}

    # --- end to end through the host-buffer API (pinned host tensors, copies timed)
    if not args.no_e2e:
        tuner = ar.LinearTuner(N, K, M, cfg, args.steps)
        pin = lambda t: t.pin_memory()
        Wh = pin(torch.from_numpy(d["W"].view(np.int16)).view(torch.bfloat16))
        Xh = pin(torch.from_numpy(d["X"].view(np.int16)).view(torch.bfloat16))
        Vh = pin(torch.zeros((N, K), dtype=torch.float32))
        ah = pin(torch.ones((N, K // g), dtype=torch.float32))
        bh = pin(torch.ones((N, K // g), dtype=torch.float32))
        lh = pin(torch.empty(args.steps, dtype=torch.float32))
        tuner.run_host(Wh, Xh, Vh.clone().pin_memory(), ah.clone().pin_memory(), bh.clone().pin_memory(), lh)
        torch.cuda.synchronize()
        Vw, aw, bw = Vh.clone().pin_memory(), ah.clone().pin_memory(), bh.clone().pin_memory()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        tuner.run_host(Wh, Xh, Vw, aw, bw, lh)
        f1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(f0.elapsed_time(f1), dist if world > 1 else None, "cuda")
        result["e2e"] = {"value": job_throughput(world, args.steps, e2e_ms), "unit": "steps/s",
                         "h2d_bytes_per_step": tuner.h2d_bytes() / args.steps,
                         "d2h_bytes_per_step": tuner.d2h_bytes() / args.steps,
                         "job": f"per layer: copy W, X, V, alpha, beta in; reference forward; {args.steps} steps; "
                                "copy V, alpha, beta and the losses out"}
        del tuner

    if rank == 0 and world == 1 and not args.no_w4a16:
        result["w4a16"] = w4a16_bench(ar, torch, peaks)
    if rank == 0 and world == 1 and not args.no_nvfp4:
        result["nvfp4_qdq"] = nvfp4_bench(ar, torch, peaks)
    if rank == 0 and world == 1 and not args.no_extra:
        del W, X, V, alpha, beta, Y, ws
        torch.cuda.empty_cache()
        result["workloads"] = other_workloads(ar, torch, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(wl, d)
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
