#!/usr/bin/env python
"""Benchmark of the ARCHead packed LM-head forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2|3|4|5] [--T T] [--impl ours|reference]

One step = one forward call of the packed head over one batch of seeded
synthetic hidden states (the whole hot path: low-rank prologue, the
vocabulary pass with its fused epilogue).  The default workload is the
Qwen3-8B-shaped head (V=151,936, d=4,096, core rank 512, INT4 group 128,
correction rank 64) decoding one token, with fp32 logits and argmax out.
The packed head (382 MB) is larger than L2 (126 MB), so every step streams
it from HBM; no L2 flush is needed between steps.

Multi-GPU: one process per GPU under torchrun; each rank serves its own batch
with its own copy of the head (replicas, no collective on the data path).
Timing is on the device with CUDA events, max over ranks.

--impl reference times the CPU oracle (float64 numpy) on the host cores, on a
bounded sample of vocabulary rows, scaled to the full head.

--build times the GPU construction of the packed head instead (Algorithm 1:
damped metric, the randomised truncated SVDs of Eq. 4 (--svd exact for the
exact ones), quantisers; fp64) from a seeded dense head of
the Qwen3-8B shape and 16,384 calibration states (the largest calibration
budget the pages report), with the oracle's builder on a slice of the head
rows as the CPU baseline.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import re
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import archead_inputs as gen  # noqa: E402

METRIC = "packed LM-head tokens/s & µs/call at V=151936,d=4096; % HBM or MMA roofline"
FALLBACK_HBM_GBS = 6650.0
CPU_SAMPLE_SECONDS = 12.0   # target length of the CPU-oracle sample behind cpu_baseline
REFERENCE_SECONDS = 120.0   # target length of a whole --impl reference run
FALLBACK_BF16_TFLOPS = 1590.0
DATASHEET_BF16_TFLOPS = 2250.0   # B200 dense bf16, nominal (NVIDIA's figure halved: theirs assumes 2:4 sparsity)

OPS = {  # config -> what one call produces
    2: dict(logits=True, argmax=True, lse=False, ce=False),
    3: dict(logits=False, argmax=True, lse=True, ce=False),
    4: dict(logits=False, argmax=True, lse=True, ce=True),
    5: dict(logits=False, argmax=True, lse=True, ce=True),
}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--config", type=int, default=2, choices=sorted(OPS))
    ap.add_argument("--T", type=int, default=None, help="override the token count of the config")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--shard-vocab", action="store_true",
                    help="vocabulary-sharded head: each rank holds a contiguous range of rows; one batch per step, "
                         "per-token partials all-gathered and merged (strong scaling); LSE / argmax / CE out")
    ap.add_argument("--sample", type=float, default=None, metavar="TEMPERATURE",
                    help="measure the sampling entry point (Gumbel-max draw per token at this temperature, "
                         "plus LSE and argmax) instead of the config's outputs")
    ap.add_argument("--variant", default="archead", choices=["archead", "naive-int4", "core-int4"],
                    help="head format: ARCHead, or one of the pages' storage-matched comparison heads "
                         "(Qwen-shaped configs only)")
    ap.add_argument("--build", action="store_true", help="time the GPU construction of the packed head")
    ap.add_argument("--build-steps", type=int, default=5)
    ap.add_argument("--build-warmup", type=int, default=3)
    ap.add_argument("--n-calib", type=int, default=16384, help="calibration states for --build")
    ap.add_argument("--svd", choices=("randomized", "exact"), default="randomized",
                    help="truncated SVDs of --build: the pages' randomised one (default) or the exact one")
    ap.add_argument("--svd-oversample", type=int, default=None, help="randomised SVD: sketch columns beyond r")
    ap.add_argument("--svd-power-iters", type=int, default=None, help="randomised SVD: subspace iteration steps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def peaks():
    """HBM GB/s, dense bf16 TFLOP/s (burst, sustained) and where they come from."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        burst = float(d["bf16_tflops"])
        return float(d["hbm_gbs"]), burst, float(d.get("bf16_tflops_sustained", burst)), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS, "fallback"


def max_over_ranks(ms, device):
    """The slowest rank's device time (ms): an all-reduce MAX over the process
    group, or ms itself when there is one process."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_step, steps, ms):
    """Whole-job tokens/s: every rank serves its own batch each step (replicas,
    weak scaling); ms is the slowest rank's time for all steps."""
    return world * tokens_per_step * steps / (ms / 1e3)


def workload(cfg, T, variant="archead"):
    """The config's workload; a --variant swaps in one of the storage-matched
    comparison heads of the same (Qwen3-8B) shape."""
    wl = gen.WORKLOADS[cfg]
    T = wl.T if T is None else T
    if variant != "archead":
        base = gen.BASELINE_SHAPES[variant]
        if (wl.shape.V, wl.shape.d) != (base.V, base.d):
            raise SystemExit(f"--variant {variant} applies to the Qwen3-8B-shaped configs (2, 3, 5)")
        wl = dataclasses.replace(wl, name=f"{wl.name} [{variant}]", shape=base)
    return wl, T


def row_bytes(shape):
    """Packed bytes per vocabulary row: INT5 core factor and its fp16 row scale,
    INT4 residual and its fp16 group scales, INT8 correction factor and its
    fp16 row scale (a rank-0 branch has no row scale to read)."""
    V, d, r_c, r_r, g, g_B = shape
    return 5 * r_c / 8 + (2 if r_c else 0) + d / 2 + 2 * d / g + r_r + (2 if r_r else 0)


def algorithmic(shape, T, op):
    """Bytes and flops of one forward call (the method's own work, no dense head)."""
    V, d, r_c, r_r, g, g_B = shape
    head = V * row_bytes(shape) + r_c * (d + 2) + r_r * (d + 2 * d / g_B)
    io = 2 * T * d + (4 * T * V if op["logits"] else 0) + 4 * T * (op["argmax"] + op["lse"] + op["ce"])
    flops = 2 * T * V * (d + r_c + r_r) + 2 * T * d * (r_c + r_r)
    return head + io, flops


def vocab_pass_bytes_per_launch(shape, nt, op, Kz):
    """Algorithmic bytes of one vocabulary-pass launch covering nt tokens: the
    per-row packed payload (V x row_bytes) + h and z of those tokens + outputs."""
    V, d = shape[0], shape[1]
    return (V * row_bytes(shape) + 2 * nt * d + 4 * nt * Kz + (4 * nt * V if op["logits"] else 0)
            + 4 * nt * (op["argmax"] + op["lse"] + op["ce"]))


def tc_pass_bytes_flops(shape, T, op):
    """Algorithmic bytes and flops of one tensor-core launch: the per-row packed
    payload read once, the fp16 activation operand [h | z] (T x Kc), the
    per-(token, 128-row tile) partials and target logits written, logits if asked."""
    V, d, r_c, r_r = shape[0], shape[1], shape[2], shape[3]
    kc = d + -(-r_c // 64) * 64 + -(-r_r // 64) * 64
    n_mt128 = -(-V // 128)
    b = (V * row_bytes(shape) + 2 * T * kc + 16 * T * n_mt128 + 4 * T + (4 * T * V if op["logits"] else 0))
    return b, 2 * T * V * (d + r_c + r_r)


KERNEL_SOURCES = {
    "decode": ("decode.cu", "device.cuh", "params.h", "layout.h"),
    "tensor_core": ("tcgemm.cu", "tcgen05.cuh", "tc_params.h", "device.cuh", "layout.h"),
}
PROFILE_STEM = {"decode": "decode_kernel", "tensor_core": "tc_kernel"}


def source_hash(kind):
    """Hash of the sources the vocabulary-pass kernel is compiled from."""
    h = hashlib.sha256()
    cs = os.path.join(ROOT, "quantized_output_head_b200", "csrc")
    for f in KERNEL_SOURCES[kind]:
        h.update(open(os.path.join(cs, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kind, cfg, T):
    """dram bytes per vocabulary-pass launch from the committed ncu summary, if
    it was taken on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", f"{PROFILE_STEM[kind]}_cfg{cfg}_T{T}.md")
    if not os.path.exists(p):
        return None
    txt = open(p).read()
    m = re.search(r"traffic_bytes_per_launch:\s*(\d+)", txt)
    s = re.search(r"source_sha256_16:\s*([0-9a-f]+)", txt)
    if not m or not s or s.group(1) != source_hash(kind):
        return None
    return int(m.group(1))


class ClockSampler:
    """SM clock and throttle reasons from NVML, sampled in a thread."""

    def __init__(self, index, period=0.005):
        self.samples, self.max_mhz, self.err = [], None, None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report no clocks
            self._nv, self.err = None, repr(e)
        self._period = period
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((mhz, rs))
            except Exception as e:
                self.err = repr(e)
                return
            time.sleep(self._period)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0, "note": self.err}
        nv = self._nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        seen = sorted({n for _, rs in self.samples for n, bit in names.items() if rs & bit})
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": seen, "samples": len(self.samples)}


# --------------------------------------------------------------- reference
def oracle_call_model(oracle, comps, shape, h_bits, small=256, large=2048):
    """(fixed seconds per oracle call, seconds per vocabulary row) from two
    timed calls on `small` and `large` rows (best of two each)."""
    def best(n):
        rows = np.arange(min(shape.V, n))
        ts = []
        for _ in range(2):
            t0 = time.perf_counter()
            oracle.logits(comps, shape.g, shape.g_B, h_bits, rows=rows)
            ts.append(time.perf_counter() - t0)
        return rows.size, min(ts)
    n1, t1 = best(small)
    n2, t2 = best(large)
    t_row = max((t2 - t1) / max(n2 - n1, 1), 1e-7)
    return max(t1 - n1 * t_row, 0.0), t_row


def run_reference(args, cfg, wl, T):
    """The CPU oracle as it stands, timed on a bounded sample of vocabulary rows."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    shape = wl.shape
    sh = (shape.V, shape.d, shape.r_c, shape.r_r, shape.g, shape.g_B)
    comps = gen.draw_components(shape, wl.head_seed_cfg)
    h_bits, targets = gen.draw_activations(shape.d, T, shape.V, cfg)
    # Each step is a bounded sample of vocabulary rows, sized so that the whole
    # --warmup + --steps run takes about REFERENCE_SECONDS.  A call of the
    # oracle has a fixed part (decoding R, B and h) and a part per row; a
    # two-size pilot separates them, and only the per-row part is scaled to V.
    t_fixed, t_row = oracle_call_model(oracle, comps, shape, h_bits)
    per_step = REFERENCE_SECONDS / max(args.steps + args.warmup, 1)
    rows = np.arange(int(min(shape.V, max(128, (per_step - t_fixed) / t_row))))
    for _ in range(args.warmup):
        oracle.logits(comps, shape.g, shape.g_B, h_bits, rows=rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.logits(comps, shape.g, shape.g_B, h_bits, rows=rows)
    dt = (time.perf_counter() - t0) / args.steps
    per_call = t_fixed + max(dt - t_fixed, 0.0) * shape.V / rows.size
    value = T / per_call
    sample = (f"{rows.size} of {shape.V} vocabulary rows x {T} tokens per step; the per-row time scaled to the "
              f"full head, the fixed {t_fixed * 1e3:.0f} ms per call counted once")
    return dict(impl="reference", metric=METRIC, value=value, unit="tokens/s", n_gpus=args.gpus,
                steps=args.steps, warmup=args.warmup, ms_per_step=per_call * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                config=dict(workload=wl.name, V=shape.V, d=shape.d, r_c=shape.r_c, r_r=shape.r_r, g=shape.g,
                            g_B=shape.g_B, T=T),
                cpu_baseline=dict(kind="oracle", value=value, unit="tokens/s", cores=cores, sample=sample),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0),
                algorithmic=dict(zip(("bytes", "flops"), algorithmic(sh, T, OPS[cfg]))))


def oracle_parity(oracle, shape, h_bits, y, rowmax, gpu):
    """The GPU outputs of the timed run against the oracle's values from the
    baseline sample: max |d logit| / tolerance on the sampled rows and, when
    the sample is the whole head, max |d LSE| / tolerance and the argmax
    mismatches beyond the tie rule (a different row is accepted only where the
    oracle's gap to it is within the two rows' tolerance)."""
    n_rows = y.shape[1]
    res = dict(rows=int(n_rows), tokens=int(y.shape[0]))
    full = n_rows == shape.V
    if gpu.get("logits") is None and not full:
        res["note"] = "sampled rows carry no GPU output to compare (no logits written)"
        return res
    tol = oracle.tolerance(h_bits, rowmax)
    if gpu.get("logits") is not None:
        res["logits_max_err_over_tol"] = float((np.abs(gpu["logits"][:, :n_rows] - y) / tol).max())
    if full:
        lse_ref, am_ref, _ = oracle.lse_argmax_ce(y)
        if gpu.get("lse") is not None:
            res["lse_max_err_over_tol"] = float((np.abs(gpu["lse"] - lse_ref) / tol.max(axis=1)).max())
        if gpu.get("argmax") is not None:
            a = gpu["argmax"].astype(np.int64)
            t = np.arange(a.size)
            inside = (a >= 0) & (a < shape.V)
            ac = np.where(inside, a, 0)
            gap = y[t, am_ref] - y[t, ac]
            bad = (a != am_ref) & (~inside | (gap > np.maximum(tol[t, ac], tol[t, am_ref])))
            res["argmax_mismatches"] = int(bad.sum())
    return res


def cpu_baseline(cfg, wl, T, comps, h_bits, gpu=None):
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    shape = wl.shape
    # A pilot on a few rows sizes the sample to about CPU_SAMPLE_SECONDS of
    # oracle work (the whole head when that fits: no scaling at all).
    pilot = min(shape.V, 2048)
    t0 = time.perf_counter()
    oracle.logits(comps, shape.g, shape.g_B, h_bits, rows=np.arange(pilot))
    t_pilot = max(time.perf_counter() - t0, 1e-3)
    n_rows = int(min(shape.V, max(pilot, pilot * CPU_SAMPLE_SECONDS / t_pilot)))
    n_rows = max(pilot, min(n_rows, int(2e9 // (8 * T))))   # at most ~2 GB of fp64 logits on the host
    rows = np.arange(n_rows)
    t0 = time.perf_counter()
    y, rowmax = oracle.logits(comps, shape.g, shape.g_B, h_bits, rows=rows)
    dt = time.perf_counter() - t0
    per_call = dt * shape.V / n_rows
    scaled = "" if n_rows == shape.V else ", scaled to the full head"
    cpu = dict(value=T / per_call, unit="tokens/s", cores=cores, kind="oracle",
               sample=f"oracle on {n_rows} of {shape.V} vocabulary rows for {T} token(s), {dt:.1f} s{scaled}")
    parity = None
    if gpu is not None:
        try:
            parity = oracle_parity(oracle, shape, h_bits, y, rowmax, gpu)
        except Exception as e:   # the check must never cost the measurement
            parity = dict(error=repr(e))
    return cpu, parity


# ------------------------------------------------------------------- build
BUILD_SHAPE = (151936, 4096, 512, 64, 128, 128)   # Qwen3-8B head: V, d, r_c, r_r, g, g_B
BUILD_ORACLE_ROWS = 4096
BUILD_OWN_KERNELS = 13    # launches of the builder's own kernels per build (the rest is cuBLAS / cuSOLVER)


def sketch_cols(d, r, oversample):
    """Columns of the randomised SVD's sketch (archead_svd_opts: r + oversample,
    rounded up to a multiple of 64 above 64, at most d)."""
    k = r + oversample
    return min(d, (k + 63) // 64 * 64 if k > 64 else k)


def build_flops(V, d, r_c, r_r, N, svd="exact", oversample=0, power_iters=0):
    """fp64 flops of the dense products of one build (eigensolvers and QR not
    counted): H^T H, W^T W, E^T E (one triangle each), A_c = W V_c, W - A_c B_c,
    E -= L_hat R_hat, A_w = E (T_p V_w), B_w, and the d x d products of T_p,
    T_p^-1 and T_p E^T E T_p; for the randomised SVDs also, per factorisation
    of rank r with k sketch columns, power_iters + 2 products G Q (d x d x k),
    the projection Q^T G Q and the Ritz vectors (d x k x k each)."""
    f = (N * d * d + 2 * V * d * d + 6 * V * d * r_c + 2 * V * d * r_r
         + 8 * d ** 3 + 4 * d * d * r_r)
    if svd == "randomized":
        for r in (r_c, r_r):
            if r > 0:
                k = sketch_cols(d, r, oversample)
                f += 2 * d * d * k * (power_iters + 2) + 4 * d * k * k
    return f


def dgemm_peak_tflops(torch, n=8192, reps=8):
    """fp64 tensor-core throughput of a plain cuBLAS DGEMM, measured here."""
    a = torch.randn(n, n, dtype=torch.float64, device="cuda")
    b = torch.randn(n, n, dtype=torch.float64, device="cuda")
    c = a @ b
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.matmul(a, b, out=c)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1) / 1e3)
    del a, b, c
    return 2 * n ** 3 / best / 1e12


def build_cpu_baseline(W, H, shape):
    """The oracle builder on the first BUILD_ORACLE_ROWS head rows (same d,
    ranks, groups and calibration states); its V-independent metric step is
    timed on its own and the rest scaled by V."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    V, d, r_c, r_r, g, g_B = shape
    Ws = W[:BUILD_ORACLE_ROWS].double().cpu().numpy()
    Hs = H.double().cpu().numpy()
    t0 = time.perf_counter()
    oracle.damped_metric(Hs, 1e-2, 0.75)
    t_metric = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.build_packed_head(Ws, Hs, r_c=r_c, r_r=r_r, g=g, g_B=g_B, p=0.75, lam=1e-2)
    t_sample = time.perf_counter() - t0
    est = t_metric + max(t_sample - t_metric, 0.0) * V / BUILD_ORACLE_ROWS
    return dict(value=est, unit="s per build", cores=cores, kind="oracle",
                sample=(f"oracle builder on {BUILD_ORACLE_ROWS} of {V} head rows ({t_sample:.1f} s, of which the "
                        f"metric {t_metric:.1f} s); the rest scaled by V (the SVDs of a {BUILD_ORACLE_ROWS} x {d} "
                        f"slice cost less per row than the full head's, so this underestimates the CPU)"))


def run_build(args):
    import torch
    import quantized_output_head_b200.builder as bld
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world != 1:
        raise SystemExit("--build runs on one GPU (each build is independent: replicas only)")
    torch.cuda.set_device(0)
    V, d, r_c, r_r, g, g_B = BUILD_SHAPE
    N = args.n_calib
    W, H = gen.dense_head_inputs_device(V, d, N)
    ws = bld.workspace(V, d, r_c, r_r, g, g_B, N)
    st = torch.cuda.current_stream()
    svd_kw = dict(svd=args.svd)
    if args.svd == "randomized":
        svd_kw.update(oversample=bld.RANDOMIZED_OVERSAMPLE if args.svd_oversample is None else args.svd_oversample,
                      power_iters=(bld.RANDOMIZED_POWER_ITERS if args.svd_power_iters is None
                                   else args.svd_power_iters))
    for _ in range(args.build_warmup):
        bld.build_head(W, H, r_c, r_r, g, g_B, ws=ws, **svd_kw)
    torch.cuda.synchronize()
    times = []
    with ClockSampler(0, period=0.05) as clk:
        for _ in range(args.build_steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            out = bld.build_head(W, H, r_c, r_r, g, g_B, ws=ws, **svd_kw)
            e1.record(st)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / 1e3)
    sec = sum(times) / len(times)
    flops = build_flops(V, d, r_c, r_r, N, svd=args.svd, oversample=svd_kw.get("oversample", 0),
                        power_iters=svd_kw.get("power_iters", 0))
    peak = dgemm_peak_tflops(torch)
    # End to end: pinned host W and H in, every packed component back to pinned host memory.
    Wh, Hh = W.cpu().pin_memory(), H.cpu().pin_memory()
    outs_h = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in out.items()}
    e_times = []
    for it in range(0 if args.no_e2e else 2):
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        Wd, Hd = Wh.cuda(non_blocking=True), Hh.cuda(non_blocking=True)
        comps = bld.build_head(Wd, Hd, r_c, r_r, g, g_B, ws=ws, **svd_kw)
        for k, v in comps.items():
            outs_h[k].copy_(v, non_blocking=True)
        torch.cuda.synchronize()
        e_times.append(time.perf_counter() - t0)
        del Wd, Hd, comps
    e_sec = min(e_times) if e_times else None
    cpu = None if args.no_cpu_baseline else build_cpu_baseline(W, H, BUILD_SHAPE)
    line = dict(
        metric="ARCHead packed-head build time (Algorithm 1) at V=151936, d=4096, r_c=512, r_r=64, N=16384",
        value=sec, unit="s per build", n_gpus=1, steps=args.build_steps, warmup=args.build_warmup,
        ms_per_step=sec * 1e3, higher_is_better=False, scaling="weak", vs_baseline=None, dtype="f64",
        data="synthetic (seeded dense head: rank-32 Gaussian part + noise; anisotropic calibration states)",
        config=dict(workload=f"qwen3-8b-head build N{N}", V=V, d=d, r_c=r_c, r_r=r_r, g=g, g_B=g_B, n_calib=N,
                    p=0.75, lam=1e-2, svd=svd_kw, parallelism="replicas x1",
                    l2="inputs larger than L2 (W 2.5 GB fp32)"),
        roofline=dict(bound="tensor", achieved=flops / sec / 1e12, peak=peak, unit="TFLOP/s",
                      frac=flops / sec / 1e12 / peak, traffic=None, kernel="whole build (cuBLAS fp64 products, "
                      "cuSOLVER eigensolvers, own kernels)", algorithmic_flops_per_launch=flops,
                      peak_source="measured here: cuBLAS DGEMM 8192^3, best of 8 (fp64 tensor cores)"),
        cpu_baseline=cpu,
        e2e=None if e_sec is None else dict(
            value=e_sec, unit="s per build", h2d_bytes_per_step=(W.numel() + H.numel()) * 4,
            d2h_bytes_per_step=sum(v.numel() * v.element_size() for v in out.values()),
            call="builder.build_head with pinned host W, H in and components out"),
        clocks=clk.summary(),
        gpu_launches=args.build_steps * (BUILD_OWN_KERNELS + (2 if args.svd == "randomized" else 0)),
        step_seconds=times)
    print(json.dumps(line))
    return 0


# -------------------------------------------------------------------- ours
def main():
    args = parse_args()
    if args.build:
        return run_build(args)
    cfg = args.config
    wl, T = workload(cfg, args.T, args.variant)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, cfg, wl, T)))
        return 0

    import torch
    import torch.distributed as dist
    import datetime
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    import quantized_output_head_b200 as qoh

    shape = wl.shape
    sh = (shape.V, shape.d, shape.r_c, shape.r_r, shape.g, shape.g_B)
    op = dict(OPS[cfg])
    comps = gen.draw_components(shape, wl.head_seed_cfg)
    h_bits, targets = gen.draw_activations(shape.d, T, shape.V, cfg)
    sharded = args.shard_vocab
    if args.sample is not None:
        if sharded:
            raise SystemExit("--sample and --shard-vocab do not combine")
        op.update(logits=False, lse=True, argmax=True, ce=False)
    if sharded:
        # This rank's rows; logits stay on their shard, the merged outputs are LSE / argmax (/ CE).
        v0, v1 = qoh.shard_rows(shape.V, world, rank)
        sh_head = (v1 - v0,) + sh[1:]
        head = qoh.PackedHead(*sh_head, qoh.shard_components(comps, v0, v1))
        head.set_vocab_shard(v0, shape.V)
        op.update(logits=False, lse=True)
    else:
        sh_head = sh
        head = qoh.PackedHead(*sh, comps)
    dev = head.device
    hd = torch.from_numpy(h_bits.view(np.int16)).to(dev)
    td = torch.from_numpy(targets).to(dev)
    logits = torch.empty((T, shape.V), dtype=torch.float32, device=dev) if op["logits"] else None
    am = torch.empty(T, dtype=torch.int32, device=dev)
    lse = torch.empty(T, dtype=torch.float32, device=dev)
    ce = torch.empty(T, dtype=torch.float32, device=dev) if op["ce"] else None
    ws = head.workspace(T)

    sample_offset = [0]

    def step():
        if args.sample is not None:
            sample_offset[0] += T   # a fresh counter range every step
            return head.sample(hd, args.sample, seed=20261202, offset=sample_offset[0])
        if sharded:
            parts = head.shard_partials(hd, td if op["ce"] else None)
            allp = qoh.gather_partials(parts) if world > 1 else parts.unsqueeze(0)
            return qoh.merge_shards(allp)
        if op["logits"]:
            head.logits_into(hd, logits, am, ws)
        else:
            head.lse_argmax_into(hd, td if op["ce"] else None, lse, am, ce, ws)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    # Timed region: K steps on the device, bracketed by barrier + synchronize.
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        ev0.record()
        for _ in range(args.steps):
            step()
        ev1.record()
        torch.cuda.synchronize()
        barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), dev)
    ms_per_step = ms / args.steps
    # Replicas: every rank serves its own batch; sharded: all ranks serve one batch.
    value = job_throughput(1 if sharded else world, T, args.steps, ms)

    # Dominant kernel (the vocabulary pass): CUDA events around it, recorded on
    # the call's stream by the library, over a second timed loop.
    kind = "decode" if args.sample is not None else head.forward_kernel(T)
    n_launch = math.ceil(T / 8) if kind == "decode" else 1
    from cuda.bindings import runtime as cudart
    _, kb = cudart.cudaEventCreate()
    _, ka = cudart.cudaEventCreate()
    head.set_profile_events(int(kb), int(ka))
    k_steps = max(10, min(args.steps, 2000))
    tot = 0.0
    for _ in range(k_steps):
        step()
        cudart.cudaEventSynchronize(ka)
        err, dt = cudart.cudaEventElapsedTime(kb, ka)
        tot += dt
    head.set_profile_events(None, None)
    cudart.cudaEventDestroy(kb)
    cudart.cudaEventDestroy(ka)
    kernel_ms = tot / k_steps / n_launch
    hbm, bf16, bf16_sust, peak_src = peaks()
    if kind == "decode":
        Kz = -(-shape.r_c // 64) * 64 + -(-shape.r_r // 32) * 32
        kbytes = vocab_pass_bytes_per_launch(sh_head, min(T, 8), op, Kz)
        kflops = None
        bound = "hbm"
    else:
        kbytes, kflops = tc_pass_bytes_flops(sh_head, T, op)
        # The roofline that binds: HBM streaming of the packed head, or the
        # tensor cores (fp16 MMA runs at the bf16 rate; sustained peak, the
        # kernel is timed inside back-to-back calls).
        bound = "tensor" if kflops / (bf16_sust * 1e12) > kbytes / (hbm * 1e9) else "hbm"
    if bound == "hbm":
        achieved, peak, unit = kbytes / (kernel_ms / 1e3) / 1e9, hbm, "GB/s"
    else:
        achieved, peak, unit = kflops / (kernel_ms / 1e3) / 1e12, bf16_sust, "TFLOP/s"
    traffic = recorded_traffic(kind, cfg, T)
    status = head.status(ws)
    launches_per_step = ((1 + n_launch) if kind == "decode" else 3) + (1 if sharded else 0)

    # End to end through the host-buffer entry point, every rank at once (each
    # serves its own batch); the slowest rank's time sets the job's figure.
    e2e = None
    if not args.no_e2e and not sharded and args.sample is None:
        # The same outputs as the timed step, through the host-buffer entry
        # point of the same operation (pinned host memory in and out).
        hh = torch.from_numpy(h_bits.view(np.int16)).pin_memory().numpy().view(np.uint16)
        th = torch.from_numpy(targets).pin_memory().numpy()
        if op["logits"]:
            outs = (torch.empty((T, shape.V), dtype=torch.float32).pin_memory().numpy(),
                    torch.empty(T, dtype=torch.int32).pin_memory().numpy())
            e2e_call = head.prepare_logits_host(hh, outs)
            h2d, d2h = T * shape.d * 2, T * shape.V * 4 + 4 * T
            what = "archead_logits_host (host buffers, fp32 logits + argmax; prepared call)"
        else:
            outs = (torch.empty(T, dtype=torch.float32).pin_memory().numpy(),
                    torch.empty(T, dtype=torch.int32).pin_memory().numpy(),
                    torch.empty(T, dtype=torch.float32).pin_memory().numpy() if op["ce"] else None)
            e2e_call = head.prepare_lse_argmax_host(hh, th if op["ce"] else None, outs)
            h2d = T * shape.d * 2 + (4 * T if op["ce"] else 0)
            d2h = 4 * T * (2 + (1 if op["ce"] else 0))
            what = ("archead_lse_argmax_host (host buffers, lse + argmax" + (" + ce" if op["ce"] else "") +
                    "; prepared call)")
        for _ in range(3):
            e2e_call()
        e_steps = max(10, min(args.steps, 2000))
        barrier()
        t0 = time.perf_counter()
        for _ in range(e_steps):
            e2e_call()
        e_ms = max_over_ranks((time.perf_counter() - t0) * 1e3, dev)
        e_dt = e_ms / 1e3 / e_steps
        e2e = dict(value=world * T / e_dt, unit="tokens/s", h2d_bytes_per_step=world * h2d,
                   d2h_bytes_per_step=world * d2h, us_per_call=e_dt * 1e6, call=what)

    out = None
    if rank == 0:
        cpu = parity = None
        if world == 1 and not args.no_cpu_baseline:
            gpu_out = None
            if not sharded and args.sample is None:   # the last timed step's outputs are in these buffers
                torch.cuda.synchronize()
                gpu_out = dict(logits=None if logits is None else logits.cpu().numpy().astype(np.float64),
                               lse=lse.cpu().numpy().astype(np.float64) if op["lse"] else None,
                               argmax=am.cpu().numpy())
            cpu, parity = cpu_baseline(cfg, wl, T, comps, h_bits, gpu_out)
        ab, af = algorithmic(sh, T, op)
        out = dict(
            metric=METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps, warmup=args.warmup,
            ms_per_step=ms_per_step, us_per_call=ms_per_step * 1e3, higher_is_better=True,
            scaling="strong" if sharded else "weak",
            vs_baseline=None, dtype="f16",
            dtype_detail=("f16 MMA (mma.sync) on exact int4/int5/int8 codes, fp32 accumulate, scales in fp32"
                          if kind == "decode" else
                          "f16 MMA (tcgen05) on fp16(scale*code) weights and fp16 [h|z], fp32 accumulate in TMEM"),
            data="synthetic (seeded, shapes of the pages' heads)",
            config=dict(workload=wl.name + (f" [sampling, temperature {args.sample}]" if args.sample is not None else ""),
                        V=shape.V, d=shape.d, r_c=shape.r_c, r_r=shape.r_r, g=shape.g,
                        g_B=shape.g_B, T=T, outputs=[k for k, v in op.items() if v] + (["sample"] if args.sample is not None else []),
                        parallelism=(f"vocabulary shards x{world} (rows {v0}-{v1} on rank 0)" if sharded
                                     else f"replicas x{world}"),
                        l2="inputs larger than L2 (packed head 382 MB)"),
            roofline=dict(bound=bound, achieved=achieved, peak=peak, unit=unit, frac=achieved / peak,
                          traffic=traffic, kernel=f"archead::{PROFILE_STEM[kind]}", kernel_us=kernel_ms * 1e3,
                          algorithmic_bytes_per_launch=kbytes, algorithmic_flops_per_launch=kflops,
                          peak_source=peak_src + ((" (sustained bf16)" if peak_src == "measured" else
                                                   " (the pool's burst bf16 figure)") if bound == "tensor" else ""),
                          **(dict(datasheet_peak=DATASHEET_BF16_TFLOPS, datasheet_frac=achieved / DATASHEET_BF16_TFLOPS)
                             if bound == "tensor" else {})),
            call=dict(algorithmic_bytes=ab, algorithmic_flops=af, gbs=ab / (ms_per_step / 1e3) / 1e9,
                      hbm_frac=ab / (ms_per_step / 1e3) / 1e9 / hbm),
            cpu_baseline=cpu, parity=parity, e2e=e2e, clocks=clk.summary(),
            gpu_launches=args.steps * launches_per_step, device_status=status,
        )
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if out is not None:
        print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
