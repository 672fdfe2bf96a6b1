#!/usr/bin/env python3
"""Benchmark of the SmoothQuant W8A8 smoothed linear layer on B200.

The measured workload is the 70B-like down projection prefill: X bf16
[8192 x 28672] with 0.05% outlier channels, W bf16 [8192 x 28672], bf16 output.
One step = one pass of the whole path over one batch, each stage a call into
libsq's C ABI on one CUDA stream:
  a1 calibrate: the activation maxima over 16 seeded calibration batches of
     2048 tokens (resident in HBM, read in one launch: the running maximum
     over batches equals the maximum over their concatenation) and the
     weight maxima, in one launch;
  a2 smoothing factors at alpha = 0.5;
  a3 fold + quantize W;  a4 smooth + quantize X;
  a5 int8 GEMM with the dequantizing epilogue.
The alpha sweep {0.25, 0.5, 0.75} (a2..a5 per alpha, after the same
calibration) is timed and reported per alpha in the same line. L2 is flushed
between steps. Other configurations (--workload) and activation variants
(--variant) serve profiling.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0). Under torchrun each rank runs an independent
replica (the path has no exchange step); value = all ranks' work / the slowest
rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from w8a8_post_quantization_calibrate_b200 import synth  # noqa: E402

METRIC = "W8A8 smoothed-linear int8 TOPS & act-quant GB/s at 1 B200; % of roofline"
WORKLOAD = "down_prefill_70b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# datasheet figures, reported beside the measured denominators for context only
SPEC_HBM_GBS = 8000.0
SPEC_INT8_TOPS = 4500.0
INT8_OVER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOP/s bf16)
L2_FLUSH_BYTES = 256 << 20
PROBE_ITERS = 4096      # one probe launch: about the length of the 70B GEMM
PROBE_LAUNCHES = 20


# ------------------------------------------------------------------ helpers
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


GEMM_SOURCES = ["w8a8_post_quantization_calibrate_b200/csrc/sq_gemm.cu",
                "w8a8_post_quantization_calibrate_b200/csrc/sq_device.cuh"]


def gemm_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    """DRAM bytes per GEMM launch from the committed ncu summary for this
    workload, or None when absent or taken on another version of the kernel
    source."""
    p = os.path.join(ROOT, "profiles", "gemm_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    per = d.get("per_workload", {}).get(workload)
    if per is None or per.get("source_sha256_16") != gemm_source_hash():
        return None
    return per.get("dram_bytes_per_launch")


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    if world > 1:
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(value: float, world: int, device) -> float:
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML while the
    timed region runs (reads only; changes no setting). mark() labels the
    samples taken from then on."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting",
               0x10: "sync_boost", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.err = None
        self.label = "setup"
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - depends on the box
            self.nvml = None
            self.err = repr(e)
        self._t = threading.Thread(target=self._run, daemon=True)

    def mark(self, label: str):
        self.label = label

    def _run(self):
        while not self._stop.is_set():
            try:
                sm = self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM)
                util = self.nvml.nvmlDeviceGetUtilizationRates(self.h).gpu
                reasons = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                pw = self.nvml.nvmlDeviceGetPowerUsage(self.h) / 1000.0
                self.samples.append((sm, util, reasons, pw, self.label))
            except Exception as e:  # pragma: no cover
                self.err = repr(e)
            self._stop.wait(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self.nvml is not None:
            self._t.join()

    def summary(self, labels=None):
        pick = [s for s in self.samples if labels is None or s[4] in labels]
        if not pick:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.err or "no samples"}
        loaded = [s for s in pick if s[1] > 0] or pick
        seen = 0
        for s in loaded:
            seen |= s[2]
        reasons = [name for bit, name in self.REASONS.items() if seen & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(s[0] for s in loaded), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(s[0] for s in loaded), "reasons": sorted(reasons), "samples": len(loaded),
                "power_w_max": round(max(s[3] for s in loaded), 1)}


def median(v):
    return statistics.median(v) if v else float("nan")


# ------------------------------------------------------------------ the CPU oracle
def _timed(fn, *a):
    t0 = time.perf_counter()
    out = fn(*a)
    return out, time.perf_counter() - t0


def oracle_stages(x_cpu, w_cpu, alpha, xcal_cpu=None, gemm_rows=256):
    """The oracle, as it stands, per stage on the workload's full tensors (a1
    over the calibration tensor and W, a2, a3 over all of W, a4 over all of X)
    and a5 on the first `gemm_rows` tokens, plus one-thread figures of a3, a4
    and a5 on bounded slices. Returns (stages dict, whole-path TOPS estimate,
    description)."""
    import oracle
    hx = synth.host_array(x_cpu)
    hw = synth.host_array(w_cpu)
    hc = hx if xcal_cpu is None else synth.host_array(xcal_cpu)
    M, K = hx.shape
    N = hw.shape[0]
    ies = x_cpu.element_size()
    threads = oracle.num_threads()
    st = {}
    xmax, t1x = _timed(oracle.col_absmax, hc)
    wmax, t1w = _timed(oracle.col_absmax, hw)
    st["a1_calibrate_xw"] = {"s": t1x + t1w, "gbs": (hc.size + hw.size) * ies / (t1x + t1w) / 1e9}
    s, t2 = _timed(oracle.smooth_factors, xmax, wmax, alpha)
    st["a2_smooth_factors"] = {"s": t2}
    (wq, wsc), t3 = _timed(oracle.fold_quant_weights, hw, s)
    st["a3_fold_quant_w"] = {"s": t3, "gbs": (hw.size * (ies + 1) + 4 * (N + K)) / t3 / 1e9}
    (xq, xsc), t4 = _timed(oracle.smooth_quant_act, hx, s)
    st["a4_smooth_quant_x"] = {"s": t4, "gbs": (hx.size * (ies + 1) + 4 * (M + K)) / t4 / 1e9}
    rows = min(gemm_rows, M)
    _, t5 = _timed(oracle.gemm_i8, np.ascontiguousarray(xq[:rows]), wq)
    t5_full = t5 * M / rows
    st["a5_w8a8_gemm"] = {"s_slice": t5, "rows": rows, "tops_slice": 2.0 * rows * N * K / t5 / 1e12,
                          "s_extrapolated": t5_full}
    # one thread, bounded slices
    oracle.set_num_threads(1)
    try:
        r1 = min(64, N)
        _, t3s = _timed(oracle.fold_quant_weights, np.ascontiguousarray(hw[:r1]), s)
        r1x = min(64, M)
        _, t4s = _timed(oracle.smooth_quant_act, np.ascontiguousarray(hx[:r1x]), s)
        r5, c5 = min(4, M), min(512, N)
        _, t5s = _timed(oracle.gemm_i8, np.ascontiguousarray(xq[:r5]), np.ascontiguousarray(wq[:c5]))
    finally:
        oracle.set_num_threads(threads)
    one = {"a3_gbs": r1 * K * (ies + 1) / t3s / 1e9, "a4_gbs": r1x * K * (ies + 1) / t4s / 1e9,
           "a5_tops": 2.0 * r5 * c5 * K / t5s / 1e12,
           "slices": f"a3 {r1} rows, a4 {r1x} rows, a5 {r5} x {c5} outputs (K={K})"}
    total = t1x + t1w + t2 + t3 + t4 + t5_full
    tops = 2.0 * M * N * K / total / 1e12
    desc = (f"oracle per stage on the full tensors (a1 over {hc.shape[0]} calibration tokens and W, a2, a3 over "
            f"W [{N} x {K}], a4 over X [{M} x {K}]) and a5 on the first {rows} tokens, extrapolated to {M}; "
            f"value = 2*{M}*{N}*{K} ops / (a1 + a2 + a3 + a4 + a5 extrapolated)")
    return {"stages": {k: {kk: (round(vv, 6) if isinstance(vv, float) else vv) for kk, vv in v.items()}
                       for k, v in st.items()},
            "one_thread": {k: (round(v, 6) if isinstance(v, float) else v) for k, v in one.items()}}, tops, desc


def oracle_slice(x: torch.Tensor, w: torch.Tensor, alpha: float, tokens: int, rows: int):
    """The whole path (a1..a5) on a tokens x rows slice (full K) -> seconds."""
    import oracle
    hx = synth.host_array(x[:tokens])
    hw = synth.host_array(w[:rows])
    t0 = time.perf_counter()
    oracle.linear(hx, hw, alpha)
    return time.perf_counter() - t0


# ------------------------------------------------------------------ our arm
def workload_inputs(name: str, decode_m: int):
    """(workload, x, w, calibration tensor or None) for a workload name;
    mlp_decode_7b takes its token count from --decode-m and uses the gate
    projection; down_prefill_70b calibrates on its 16 batches of 2048 tokens."""
    wl = synth.WORKLOADS[name]
    xcal = None
    if name == "mlp_decode_7b":
        x, w = synth.make_decode(decode_m, "gate")
    else:
        x, w = synth.make(name)
    if name == "down_prefill_70b":
        xcal = torch.cat(list(synth.calibration_batches(name)))
    return wl, x, w, xcal


VARIANTS = {
    "smoothquant": "a1(calibration X)+a1(W) in one launch, a2, a3 and a4 (one launch where the streamed row kernel "
                   "takes both tensors), a5: per-token dynamic activation scales (O1)",
    "smoothquant_steps": "a1(X) a1(W) a2 a3 a4 a5, one launch per step (per-step timings)",
    "per_tensor_dynamic": "a1(X) a1(W) a2 a3, per-tensor range of X/s, per-tensor codes, a5 (O2)",
    "per_tensor_static": "a1(X) a1(W) a2 a3, static range from the calibration maxima, per-tensor codes, a5 (O3)",
    "rmsnorm": "a1(X) a1(W) a2 a3, gain fold, RMSNorm + per-token codes, a5 (the norm-folded O1)",
    "split": "a1(X), outlier split, bulk int8 of W and X, outlier gathers, int8 GEMM + fp32 outlier epilogue",
    "fp8": "a1(X)+a1(W) in one launch, a2, a3+a4 in one launch with FP8 E4M3 codes, the FP8 GEMM (fp32 "
           "accumulation)",
    "alpha_search": "one sq_alpha_search call: a1(X) a1(W), the float reference product, then per alpha "
                    "a2 a3 a4 a5 (fp32 out) and the error reduction",
}
# the stage whose throughput the line reports as act_quant_gbs (the first present)
ACT_QUANT_STAGES = ("a4_smooth_quant_x", "a34_fold_smooth_quant_wx", "quant_per_tensor_x", "rmsnorm_quant_x",
                    "quant_bulk_x", "a34_fold_smooth_quant_wx_e4m3")
SPLIT_THRESHOLD = 6.0  # outlier channels: calibration maximum >= 6 (the synthetic outliers are 20-80x)


def pair_fits(K: int) -> bool:
    """Whether the streamed row kernel takes a3 and a4 in one launch at this K
    (both multiplier tables beside the ring); at K = 28672 they do not, and the
    pair call makes the two launches, so the step lists them separately."""
    return K <= 16384


def build_step(variant, sq, wl, x, w, xcal, dev, stream):
    """Buffers and the ordered stages of one step: [(name, callable, algorithmic
    bytes, ops)]. Every callable is one C ABI call on `stream`."""
    M, K = x.shape
    N = w.shape[0]
    C = xcal.shape[0]
    in_es = x.element_size()
    out_es = torch.empty(0, dtype=wl.out_dtype).element_size()
    maxima = torch.zeros(2 * K + 4, dtype=torch.float32, device=dev)   # xmax | wmax | amax, cleared per step
    xmax, wmax, amax = maxima[:K], maxima[K:2 * K], maxima[2 * K:2 * K + 1]
    s = torch.empty(K, dtype=torch.float32, device=dev)
    wq = torch.empty((N, K), dtype=torch.int8, device=dev)
    wsc = torch.empty(N, dtype=torch.float32, device=dev)
    xq = torch.empty((M, K), dtype=torch.int8, device=dev)
    xsc = torch.empty(M, dtype=torch.float32, device=dev)
    y = torch.empty((M, N), dtype=wl.out_dtype, device=dev)
    gws = sq.gemm_workspace(M, N, K, dev)
    ops = 2.0 * M * N * K
    gemm_bytes = M * K + N * K + M * 4 + N * 4 + M * N * out_es
    a3_bytes = N * K * in_es + K * 4 + N * K + N * 4
    act_bytes = M * K * in_es + K * 4 + M * K + M * 4
    bufs = dict(maxima=maxima, xmax=xmax, wmax=wmax, s=s, wq=wq, wsc=wsc, xq=xq, xsc=xsc, y=y, gws=gws)
    st = []
    if variant == "alpha_search":
        alphas = list(synth.DOWN_70B_ALPHAS)
        sws = torch.zeros(sq.sq_alpha_search_workspace_size(M, N, K, len(alphas)), dtype=torch.uint8, device=dev)
        once = M * K * in_es + N * K * in_es + 8 * K + (M * K + N * K) * in_es + 4 * M * N
        per_alpha = (12 * K + N * K * in_es + N * K + 4 * N + M * K * in_es + M * K + 4 * M
                     + M * K + N * K + 4 * (M + N) + 4 * M * N + 8 * M * N)
        result = {}

        def search():
            errs, best = sq.sq_alpha_search(x, w, alphas, workspace=sws, stream=stream)
            result.update(errors=[round(e, 6) for e in errs], best_alpha=best)
        st.append(("alpha_search", search, once + len(alphas) * per_alpha, len(alphas) * ops))
        return bufs, st, {"alphas": alphas, "search": result,
                          "note": "the call synchronizes its stream; ops = int8 GEMM ops over all alphas"}
    a1_pair = ("a1_calibrate_xw", lambda: sq.sq_calibrate_absmax_pair(xcal, w, xmax, wmax, stream=stream),
               (C + N) * K * in_es + 2 * K * 4, 0)
    a2 = ("a2_smooth_factors", lambda: sq.sq_smooth_factors(xmax, wmax, wl.alpha, 1e-8, s=s, stream=stream),
          3 * K * 4, 0)
    a5 = ("a5_w8a8_gemm", lambda: sq.sq_w8a8_gemm(xq, xsc, wq, wsc, y=y, workspace=gws, stream=stream),
          gemm_bytes, ops)
    if variant == "fp8":
        wq8 = torch.empty((N, K), dtype=torch.uint8, device=dev)
        xq8 = torch.empty((M, K), dtype=torch.uint8, device=dev)
        st += [a1_pair, a2]
        st.append(("a34_fold_smooth_quant_wx_e4m3",
                   lambda: sq.sq_fold_smooth_quant_pair_e4m3(w, x, s, wq=wq8, w_scale=wsc, xq=xq8, x_scale=xsc,
                                                             stream=stream),
                   (N + M) * K * in_es + K * 4 + (N + M) * K + (N + M) * 4, 0))
        st.append(("a5_w8a8_gemm", lambda: sq.sq_w8a8_gemm_e4m3(xq8, xsc, wq8, wsc, y=y, stream=stream),
                   gemm_bytes, ops))
        return bufs, st, {"note": "FP8 E4M3 codes; the GEMM kernel is the paired-SM tcgen05 kernel with "
                                  "kind::f8f6f4 operands"}
    if variant == "smoothquant":
        st += [a1_pair, a2]
        if pair_fits(K):
            st.append(("a34_fold_smooth_quant_wx",
                       lambda: sq.sq_fold_smooth_quant_pair(w, x, s, wq=wq, w_scale=wsc, xq=xq, x_scale=xsc,
                                                            stream=stream),
                       (N + M) * K * in_es + K * 4 + (N + M) * K + (N + M) * 4, 0))
        else:
            st.append(("a3_fold_quant_w", lambda: sq.sq_fold_quant_weights(w, s, wq=wq, w_scale=wsc, stream=stream),
                       a3_bytes, 0))
            st.append(("a4_smooth_quant_x", lambda: sq.sq_smooth_quant_act(x, s, xq=xq, x_scale=xsc, stream=stream),
                       act_bytes, 0))
        st.append(a5)
        return bufs, st, {}
    st.append(("a1_calibrate_x", lambda: sq.sq_calibrate_absmax(xcal, xmax, stream=stream), C * K * in_es + K * 4, 0))
    if variant == "split":
        keep = torch.empty(K, dtype=torch.float32, device=dev)
        idx = torch.empty(K, dtype=torch.int32, device=dev)
        count = torch.empty(1, dtype=torch.int32, device=dev)
        # the outlier set is static: its size is fixed once, from this workload's calibration
        sq.sq_calibrate_absmax(xcal, xmax, stream=stream)
        _, _, c0 = sq.sq_outlier_split(xmax, SPLIT_THRESHOLD, stream=stream)
        n_out = int(c0.item())
        ld = max(4, (n_out + 3) // 4 * 4)
        xo = torch.empty((M, ld), dtype=torch.float32, device=dev)
        wo = torch.empty((N, ld), dtype=torch.float32, device=dev)

        st.append(("outlier_split", lambda: sq.sq_outlier_split(xmax, SPLIT_THRESHOLD, keep=keep, idx=idx, count=count,
                                                                stream=stream), K * 4 * 2 + K * 4, 0))
        st.append(("quant_bulk_w", lambda: sq.sq_quant_bulk(w, keep, q=wq, scale=wsc, stream=stream), a3_bytes, 0))
        st.append(("quant_bulk_x", lambda: sq.sq_quant_bulk(x, keep, q=xq, scale=xsc, stream=stream), act_bytes, 0))
        st.append(("gather_x", lambda: sq.sq_gather_columns(x, idx, n_out, ld, out=xo, stream=stream),
                   M * n_out * in_es + M * ld * 4, 0))
        st.append(("gather_w", lambda: sq.sq_gather_columns(w, idx, n_out, ld, out=wo, stream=stream),
                   N * n_out * in_es + N * ld * 4, 0))
        st.append(("a5_w8a8_gemm", lambda: sq.sq_w8a8_gemm_split(xq, xsc, wq, wsc, xo, wo, y=y, workspace=gws,
                                                                  stream=stream),
                   gemm_bytes + (M + N) * ld * 4, ops))
        return bufs, st, {"outlier_channels": n_out, "ld": ld, "threshold": SPLIT_THRESHOLD}
    st.append(("a1_calibrate_w", lambda: sq.sq_calibrate_absmax(w, wmax, stream=stream), N * K * in_es + K * 4, 0))
    st.append(a2)
    st.append(("a3_fold_quant_w", lambda: sq.sq_fold_quant_weights(w, s, wq=wq, w_scale=wsc, stream=stream),
               a3_bytes, 0))
    extra = {}
    if variant == "smoothquant_steps":
        st.append(("a4_smooth_quant_x", lambda: sq.sq_smooth_quant_act(x, s, xq=xq, x_scale=xsc, stream=stream),
                   act_bytes, 0))
    elif variant == "per_tensor_dynamic":
        st.append(("tensor_absmax_x", lambda: sq.sq_tensor_absmax(x, s, amax, stream=stream),
                   M * K * in_es + K * 4 + 4, 0))
        st.append(("quant_per_tensor_x", lambda: sq.sq_quant_act_per_tensor(x, s, amax, xq=xq, x_scale=xsc,
                                                                            stream=stream),
                   act_bytes, 0))
    elif variant == "per_tensor_static":
        st.append(("static_range", lambda: sq.sq_tensor_absmax(xmax.view(1, K), s, amax, stream=stream),
                   2 * K * 4 + 4, 0))
        st.append(("quant_per_tensor_x", lambda: sq.sq_quant_act_per_tensor(x, s, amax, xq=xq, x_scale=xsc,
                                                                            stream=stream),
                   act_bytes, 0))
    elif variant == "rmsnorm":
        gain = torch.from_numpy(np.random.default_rng(0).uniform(0.5, 1.5, K).astype(np.float32)).to(dev)
        gf = torch.empty(K, dtype=torch.float32, device=dev)
        st.append(("fold_norm_gain", lambda: sq.sq_fold_norm_gain(gain, s, gain_folded=gf, stream=stream),
                   3 * K * 4, 0))
        st.append(("rmsnorm_quant_x", lambda: sq.sq_rmsnorm_quant_act(x, gf, 1e-5, xq=xq, x_scale=xsc,
                                                                      want_inv_rms=False, stream=stream),
                   act_bytes, 0))
        extra = {"norm_eps": 1e-5, "note": "x plays the hidden state; s from its maxima (kernel cost is "
                                           "independent of the values of s)"}
    st.append(a5)
    return bufs, st, extra


def int8_probe(sq, dev, stream, clk, launches=PROBE_LAUNCHES, iters=PROBE_ITERS):
    """The int8 tensor-core rate (sq_probe_tensor_int8), median over launches
    with CUDA events on the launching stream, and the SM clock each launch ran
    at (cycles over nanoseconds, measured by the kernel on one SM) -> dict."""
    clk.mark("probe")
    times, mhz, ops = [], [], 0.0
    clocks = torch.zeros(2, dtype=torch.int64, device=dev)
    for i in range(launches + 3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ops = sq.sq_probe_tensor_int8(iters, clocks=clocks, stream=stream)
        b.record(stream)
        b.synchronize()
        if i >= 3:
            times.append(a.elapsed_time(b))
            cyc, ns = (int(v) for v in clocks.tolist())
            mhz.append(1e3 * cyc / ns if ns > 0 else float("nan"))
    ms = median(times)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    tops = ops / (ms * 1e-3) / 1e12
    f = median(mhz)
    return {"tops": tops, "ms": ms, "ops_per_launch": ops, "launches": launches, "sm_mhz_measured": round(f, 1),
            "ops_per_sm_cycle": round(tops * 1e12 / (sms * f * 1e6), 1),
            "instruction": "tcgen05.mma.cta_group::2.kind::i8 256x256x32 from shared memory, every SM pair"}


def gemm_sustained(stages, stream, clk, launches=30):
    """The step's GEMM alone, back to back for `launches` launches, with the
    SM clock sampled meanwhile (the clock the GEMM runs at under its own power
    draw) -> (median ms per launch, clock summary)."""
    fn = [f for n, f, _, _ in stages if n == "a5_w8a8_gemm"][0]
    fn()
    torch.cuda.synchronize()
    clk.mark("gemm")
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(launches + 1)]
    ev[0].record(stream)
    for i in range(launches):
        fn()
        ev[i + 1].record(stream)
    ev[-1].synchronize()
    clk.mark("between")
    return median([ev[i].elapsed_time(ev[i + 1]) for i in range(launches)]), clk.summary({"gemm"})


def int_mm_probe(dev, stream, n=8192, reps=10):
    """torch._int_mm (a library int8 GEMM) at n^3, best of `reps`, as context."""
    try:
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=dev)
        for _ in range(2):
            torch._int_mm(a, b)
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            torch._int_mm(a, b)
            e1.record(stream)
            e1.synchronize()
            best = min(best, e0.elapsed_time(e1))
        return {"tops": 2.0 * n ** 3 / (best * 1e-3) / 1e12, "ms": round(best, 4), "shape": f"{n}^3"}
    except Exception as e:  # pragma: no cover - depends on the box
        return {"unavailable": repr(e)[:200]}


def run_ours(args, world, rank, local):
    from w8a8_post_quantization_calibrate_b200 import sq
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    init_dist(world, "nccl")
    wl, x_cpu, w_cpu, xcal_cpu = workload_inputs(args.workload, args.decode_m)
    M, K = x_cpu.shape
    N = w_cpu.shape[0]
    x = x_cpu.to(dev)
    w = w_cpu.to(dev)
    xcal = x if xcal_cpu is None else xcal_cpu.to(dev)
    in_es, out_es = x_cpu.element_size(), torch.empty(0, dtype=wl.out_dtype).element_size()
    stream = torch.cuda.current_stream(dev)

    bufs, stages, variant_info = build_step(args.variant, sq, wl, x, w, xcal, dev, stream)
    maxima = bufs["maxima"]
    names = [n for n, _, _, _ in stages]
    nst = len(stages)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_read = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        # Evict the step's operands from L2: write 256 MiB, then read another
        # 256 MiB so that no dirty lines are left whose write-back the next
        # kernel would pay for.
        flush.zero_()
        flush_read.amax()

    def step(ev=None):
        maxima.zero_()
        for j, (_, fn, _, _) in enumerate(stages):
            if ev: ev[j].record(stream)
            fn()
        if ev: ev[nst].record(stream)

    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize(dev)
    if sq.sq_get_status(stream) != sq.SQ_OK:
        raise RuntimeError("device status error during warm-up")

    # Timed region: K steps with one event pair each (no events between the
    # kernels, so consecutive launches overlap as they do in use: every kernel
    # is launched with programmatic dependent launch).
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
    # A second, instrumented pass (events between the kernels) gives each
    # kernel's duration for the kernel table and the roofline.
    n_inst = max(args.steps, args.kernel_steps)
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nst + 1)] for _ in range(n_inst)]
    sweep = None
    with ClockSampler(dev.index if dev.index is not None else 0) as clk:
        barrier(world)
        torch.cuda.synchronize(dev)
        clk.mark("steps")
        for i in range(args.steps):
            flush_l2()
            step_ev[i][0].record(stream)
            step()
            step_ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        clk.mark("between")
        barrier(world)
        clk.mark("kernels")
        for i in range(n_inst):
            flush_l2()
            step(events[i])
        torch.cuda.synchronize(dev)
        clk.mark("between")
        if args.variant == "smoothquant" and args.sweep_steps > 0 and wl.name == "down_prefill_70b":
            clk.mark("sweep")
            sweep = alpha_sweep(sq, bufs, stages, x, w, stream, flush_l2, args.sweep_steps)
            clk.mark("between")
        probe = int8_probe(sq, dev, stream, clk) if M > 16 and args.variant != "alpha_search" else None
        clk.mark("between")
        sustained = (gemm_sustained(stages, stream, clk) if M > 16 and args.variant != "alpha_search"
                     else (None, None))
    barrier(world)
    status = sq.sq_get_status(stream)
    if status != sq.SQ_OK:
        raise RuntimeError(f"device status {status} after the timed region")

    step_times = [a.elapsed_time(b) for a, b in step_ev]
    step_ms = median(step_times)
    per_kernel = {n: median([ev[j].elapsed_time(ev[j + 1]) for ev in events]) for j, n in enumerate(names)}
    inst_step_ms = median([ev[0].elapsed_time(ev[nst]) for ev in events])
    step_ms_max = max_over_ranks(step_ms, world, dev)
    ops = 2.0 * M * N * K
    value = world * ops / (step_ms_max * 1e-3) / 1e12

    peaks, peak_src = load_peaks()
    bf16_peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    int8_from_bf16 = bf16_peak * INT8_OVER_BF16
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    int8_peak = probe["tops"] if probe else int8_from_bf16
    kb = {n: b for n, _, b, _ in stages}
    kernels = {}
    for n in names:
        ms = per_kernel[n]
        entry = {"ms": round(ms, 5), "gbs": round(kb[n] / (ms * 1e-3) / 1e9, 1),
                 "hbm_frac": round(kb[n] / (ms * 1e-3) / 1e9 / hbm, 3),
                 "hbm_frac_of_spec": round(kb[n] / (ms * 1e-3) / 1e9 / SPEC_HBM_GBS, 3)}
        if n == "a5_w8a8_gemm":
            tops = ops / (ms * 1e-3) / 1e12
            entry.update({"tops": round(tops, 1), "tensor_frac": round(tops / int8_peak, 3),
                          "tensor_frac_of_bf16x2": round(tops / int8_from_bf16, 3),
                          "tensor_frac_of_spec": round(tops / SPEC_INT8_TOPS, 3)})
        kernels[n] = entry
    clocks_k = clk.summary({"kernels"})
    clocks_p = clk.summary({"probe"})
    if args.variant == "alpha_search":
        ms = per_kernel["alpha_search"]
        n_a = len(variant_info["alphas"])
        value = world * n_a * ops / (step_ms_max * 1e-3) / 1e12
        gbs = kb["alpha_search"] / (ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": "the whole search (memory-bound passes dominate; the int8 and "
                                              "reference GEMMs are included in the time)",
                    "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                    "traffic": None, "peak_source": f"{peak_src}: hbm_gbs",
                    "algorithmic_bytes_per_launch": kb["alpha_search"]}
        kernels["alpha_search"]["per_alpha_ms"] = round(ms / n_a, 4)
    elif M > 16:
        gemm_ms = per_kernel["a5_w8a8_gemm"]
        achieved = ops / (gemm_ms * 1e-3) / 1e12
        default_gemm = args.variant not in ("split", "fp8")
        roofline = {"bound": "tensor", "kernel": ("gemm_pair_kernel (a5, paired-SM tcgen05)" if M > 128
                                                  else "gemm_tiled_kernel (a5)")
                    + (", FP8 E4M3 operands" if args.variant == "fp8" else ""),
                    "achieved": round(achieved, 1), "peak": round(int8_peak, 1), "unit": "TOPS",
                    "frac": round(achieved / int8_peak, 4),
                    "traffic": load_traffic(args.workload) if (M > 128 and default_gemm) else None,
                    "peak_source": ("measured int8: sq_probe_tensor_int8 in this run (median of "
                                    f"{probe['launches']} launches of {probe['ms']:.3f} ms at "
                                    f"{probe['sm_mhz_measured']} MHz measured in the kernel); SM clock median "
                                    f"{clocks_k.get('sm_mhz')} MHz (NVML) during the kernel pass" if probe else
                                    f"{peak_src}: bf16 x {INT8_OVER_BF16}"),
                    "peak_bf16x2": round(int8_from_bf16, 1),
                    "frac_of_bf16x2": round(achieved / int8_from_bf16, 4),
                    "bf16x2_source": f"{peak_src}: bf16 {bf16_peak} TFLOP/s (burst) x {INT8_OVER_BF16} nominal "
                                     f"int8/bf16 ratio",
                    "peak_spec": SPEC_INT8_TOPS, "frac_of_spec": round(achieved / SPEC_INT8_TOPS, 4),
                    "algorithmic_ops_per_launch": ops}
        if probe and sustained[0] and sustained[1].get("sm_mhz"):
            # per clock: the GEMM's ops per SM cycle (its back-to-back time at the
            # clock sampled while it alone ran) over the probe's (its own clock)
            sms = torch.cuda.get_device_properties(dev).multi_processor_count
            g_tops = ops / (sustained[0] * 1e-3) / 1e12
            g_opc = g_tops * 1e12 / (sms * sustained[1]["sm_mhz"] * 1e6)
            roofline["per_clock"] = {"gemm_back_to_back_ms": round(sustained[0], 5), "gemm_tops": round(g_tops, 1),
                                     "gemm_sm_mhz": sustained[1]["sm_mhz"], "gemm_ops_per_sm_cycle": round(g_opc, 1),
                                     "probe_ops_per_sm_cycle": probe["ops_per_sm_cycle"],
                                     "frac": round(g_opc / probe["ops_per_sm_cycle"], 4),
                                     "gemm_clock_reasons": sustained[1].get("reasons")}
    else:
        gemm_ms = per_kernel["a5_w8a8_gemm"]
        gbs = kb["a5_w8a8_gemm"] / (gemm_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": "gemm_stream_kernel (a5, split-K weight streaming)",
                    "achieved": round(gbs, 1), "peak": hbm, "unit": "GB/s", "frac": round(gbs / hbm, 4),
                    "traffic": None, "peak_source": f"{peak_src}: hbm_gbs",
                    "algorithmic_bytes_per_launch": kb["a5_w8a8_gemm"]}

    # end to end through the public API: pinned host X and W in, host Y out
    e2e = None
    if args.e2e_steps > 0 and args.variant == "smoothquant":
        xh = x_cpu.pin_memory()
        wh = w_cpu.pin_memory()
        yh = torch.empty((M, N), dtype=wl.out_dtype).pin_memory()
        lws = torch.zeros(sq.sq_linear_workspace_size(M, N, K, x_cpu.dtype, wl.out_dtype), dtype=torch.uint8,
                          device=dev)
        for _ in range(2):
            sq.sq_linear(xh, wh, wl.alpha, out_dtype=wl.out_dtype, y=yh, workspace=lws, stream=stream)
        torch.cuda.synchronize(dev)
        # K calls back to back: a call's input copies overlap the previous
        # call's GEMM and output copy, as in a stream of batches.
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        e_start.record(stream)
        for _ in range(args.e2e_steps):
            sq.sq_linear(xh, wh, wl.alpha, out_dtype=wl.out_dtype, y=yh, workspace=lws, stream=stream)
        e_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / args.e2e_steps, world, dev)
        e2e = {"value": round(world * ops / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TOPS",
               "ms_per_step": round(e2e_ms, 3),
               "h2d_bytes_per_step": x_cpu.numel() * in_es + w_cpu.numel() * in_es,
               "d2h_bytes_per_step": M * N * out_es,
               "api": "sq_linear (C ABI) with pinned host buffers, calls back to back (each call's input copies "
                      "overlap the previous call's GEMM and output copy); sq_linear calibrates on its own batch"}
        del xh, wh, yh, lws

    int_mm = int_mm_probe(dev, stream) if (M > 16 and args.int_mm) else None

    cpu_baseline = None
    if rank == 0 and world == 1 and args.cpu_baseline and args.variant == "smoothquant":
        import oracle
        per, tops_cpu, desc = oracle_stages(x_cpu, w_cpu, wl.alpha, xcal_cpu)
        cpu_baseline = {"value": round(tops_cpu, 6), "unit": "TOPS", "cores": oracle.num_threads(),
                        "kind": "oracle", "sample": desc, "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                        **per}
        if args.workload != "qkv_prefill_7b":
            _, xq7, wq7, _ = workload_inputs("qkv_prefill_7b", 16)
            per7, tops7, _ = oracle_stages(xq7, wq7, synth.WORKLOADS["qkv_prefill_7b"].alpha)
            cpu_baseline["qkv_prefill_7b"] = {"tops": round(tops7, 6), **per7}

    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return None
    launches = nst   # one launch of this library per stage
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_ms_max, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded outlier-bearing activations, N(0, 1/sqrt(K)) weights)",
        "config": {"workload": args.workload, "M": M, "N": N, "K": K,
                   "in_dtype": str(x_cpu.dtype).replace("torch.", ""),
                   "out_dtype": str(wl.out_dtype).replace("torch.", ""),
                   "alpha": wl.alpha,
                   "calibration": (f"{xcal.shape[0] // synth.DOWN_70B_CALIB_TOKENS} batches x "
                                   f"{synth.DOWN_70B_CALIB_TOKENS} tokens, resident, one launch"
                                   if xcal_cpu is not None else "the step's own batch"),
                   "l2": "flushed between steps (256 MiB write, then 256 MiB read)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "variant": args.variant, "step": VARIANTS[args.variant] + ", one stream", **variant_info,
                   "timing": f"value: median of {args.steps} steps with one CUDA event pair each (mean "
                             f"{round(sum(step_times) / len(step_times), 5)} ms); kernel table: medians over "
                             f"{n_inst} further steps with events between the kernels (the step there "
                             f"{round(inst_step_ms, 5)} ms: events between kernels stop the launches' overlap)"},
        "act_quant_gbs": next((kernels[n]["gbs"] for n in ACT_QUANT_STAGES if n in kernels), None),
        "act_quant_gbs_from": next((n for n in ACT_QUANT_STAGES if n in kernels), None),
        "roofline": roofline, "kernels": kernels, "cpu_baseline": cpu_baseline, "e2e": e2e,
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary({"steps", "kernels", "sweep"}),
        "clocks_by_phase": {p: clk.summary({p}) for p in ("steps", "kernels", "sweep", "probe", "gemm")},
    }
    if probe:
        out["int8_probe"] = {k: (round(v, 4) if isinstance(v, float) else v) for k, v in probe.items()}
    if int_mm:
        out["int_mm_context"] = int_mm
    if sweep:
        out["alpha_sweep"] = sweep
    return out


def alpha_sweep(sq, bufs, stages, x, w, stream, flush_l2, steps):
    """Per alpha in {0.25, 0.5, 0.75}: a2, a3, a4 and a5 after the step's
    calibration (the maxima of the last step stay in place), timed per stage
    with CUDA events, medians over `steps` repetitions; plus the codes'
    agreement check that the three alphas give three different weight sets."""
    xmax, wmax, s = bufs["xmax"], bufs["wmax"], bufs["s"]
    wq, wsc, xq, xsc, y, gws = bufs["wq"], bufs["wsc"], bufs["xq"], bufs["xsc"], bufs["y"], bufs["gws"]
    # calibration once (the sweep reuses it)
    bufs["maxima"].zero_()
    stages[0][1]()
    M, K = x.shape
    N = w.shape[0]
    ops = 2.0 * M * N * K
    out = {}
    w_checksums = []
    for a in synth.DOWN_70B_ALPHAS:
        fns = [("a2", lambda: sq.sq_smooth_factors(xmax, wmax, a, 1e-8, s=s, stream=stream)),
               ("a3", lambda: sq.sq_fold_quant_weights(w, s, wq=wq, w_scale=wsc, stream=stream)),
               ("a4", lambda: sq.sq_smooth_quant_act(x, s, xq=xq, x_scale=xsc, stream=stream)),
               ("a5", lambda: sq.sq_w8a8_gemm(xq, xsc, wq, wsc, y=y, workspace=gws, stream=stream))]
        times = {n: [] for n, _ in fns}
        tot = []
        for i in range(steps + 2):
            flush_l2()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
            for j, (_, fn) in enumerate(fns):
                ev[j].record(stream)
                fn()
            ev[-1].record(stream)
            ev[-1].synchronize()
            if i >= 2:
                for j, (n, _) in enumerate(fns):
                    times[n].append(ev[j].elapsed_time(ev[j + 1]))
                tot.append(ev[0].elapsed_time(ev[-1]))
        w_checksums.append(float(wsc.double().sum().item()))
        ms = median(tot)
        out[str(a)] = {"ms": round(ms, 5), "tops": round(ops / (ms * 1e-3) / 1e12, 1),
                       **{f"{n}_ms": round(median(v), 5) for n, v in times.items()}}
    out["distinct_weight_scales"] = len(set(w_checksums)) == len(w_checksums)
    out["note"] = (f"a2..a5 per alpha after the step's calibration, medians of {steps} repetitions with events "
                   "between the stages, L2 flushed before each")
    return out


# ------------------------------------------------------------------ reference arm
def run_reference(args, world, rank):
    """The oracle (plain C on the host cores) on this workload, as the
    reference arm: each step is one bounded sample of the workload (the whole
    path on a slice of tokens x output channels, full K)."""
    if rank != 0:
        return None
    import oracle
    wl = synth.WORKLOADS[args.workload]
    if args.workload == "mlp_decode_7b":
        x_cpu, w_cpu = synth.make_decode(args.decode_m, "gate")
    else:
        # the slice the arm times is all it needs: draw only those rows
        x_cpu = synth.activations(min(64, wl.T), wl.K, wl.outliers, wl.seed, wl.in_dtype)
        w_cpu = synth.weights(min(256, wl.N), wl.K, wl.w_std, wl.seed, wl.in_dtype)
    if args.workload == "mlp_decode_7b":
        M, K, N = x_cpu.shape[0], x_cpu.shape[1], w_cpu.shape[0]
    else:
        M, K, N = wl.T, wl.K, wl.N
    budget = max(0.002, args.reference_budget_s / max(1, args.steps + args.warmup))
    tokens, rows = min(64, x_cpu.shape[0]), min(256, w_cpu.shape[0])
    per = oracle_slice(x_cpu, w_cpu, wl.alpha, tokens, rows)
    while per > budget and tokens > 1:
        tokens //= 2
        per /= 2
    for _ in range(args.warmup):
        oracle_slice(x_cpu, w_cpu, wl.alpha, tokens, rows)
    el = 0.0
    for _ in range(args.steps):
        el += oracle_slice(x_cpu, w_cpu, wl.alpha, tokens, rows)
    ops = 2.0 * tokens * rows * K
    value = ops * args.steps / el / 1e12
    desc = (f"oracle whole path (a1..a5) on a {tokens}-token x {rows}-output-channel slice of the "
            f"workload per step (K={K}); value = int8 ops of the slice / time; {cpu_model()}, "
            f"{os.cpu_count()} logical CPUs")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic", "config": {"workload": args.workload, "M": M, "N": N, "K": K,
                                        "in_dtype": str(x_cpu.dtype).replace("torch.", ""),
                                        "out_dtype": str(wl.out_dtype).replace("torch.", ""), "alpha": wl.alpha},
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(synth.WORKLOADS), default=WORKLOAD,
                    help="the measured configuration is the 70B down projection prefill; the others are for "
                         "profiling")
    ap.add_argument("--decode-m", type=int, default=16, choices=synth.DECODE_MS)
    ap.add_argument("--variant", choices=sorted(VARIANTS), default="smoothquant",
                    help="the measured path is smoothquant (per-token O1); the others measure the other "
                         "activation granularities, the norm-folded form and the outlier decomposition")
    ap.add_argument("--kernel-steps", type=int, default=100, help="steps of the instrumented (per-kernel) pass")
    ap.add_argument("--sweep-steps", type=int, default=10, help="repetitions per alpha of the alpha sweep")
    ap.add_argument("--e2e-steps", type=int, default=5, help="steps of the end-to-end measurement")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false",
                    help="skip the oracle's per-stage timing on the host cores")
    ap.add_argument("--no-int-mm", dest="int_mm", action="store_false",
                    help="skip the torch._int_mm context figure")
    ap.add_argument("--reference-budget-s", type=float, default=90.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world != args.gpus and world > 1:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    if args.impl == "reference":
        out = run_reference(args, world, rank)
    else:
        out = run_ours(args, world, rank, local)
    if out is not None:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
