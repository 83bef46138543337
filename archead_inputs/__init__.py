"""Seeded synthetic inputs for the ARCHead packed LM-head forward.

This module is shared by the CPU oracle side (tests, ``oracle/``) and the GPU
side (tests, ``bench.py``, ``__graft_entry__``).  It holds NO arithmetic of the
method: only shapes, random draws, and the IEEE encodings (bf16 / fp16 bit
patterns) of the values it draws.  Everything the method computes (dequantising,
multiplying, quantising a dense head, the activation metric, log-sum-exp, ...)
lives either in ``oracle/`` or in the CUDA library, never here.

Workloads (ARCHead: Activation-Metric Residual Correction for Large Language
Model Output Heads, §1 and §3.3): the pages evaluate a Qwen3-8B-Base head of
151,936 x 4,096 and a Gemma-4-E4B head; neither the weights nor the calibration
text are available, so every input below is a seeded stand-in with the pages'
shapes.  Hidden states are anisotropic Gaussians, because the method exists to
exploit anisotropic final hidden states (§1, §3.1).

Draw order for every config (fixed, so a config is reproducible from its seed):
  activation stream, seed 20260802 + cfg:  basis Q0 -> h -> targets
  component stream, seed 20260802 + 100 + head:  L, s_L -> R, s_R -> q, s_res -> A, s_A -> B, s_B
The Qwen-shaped configs 2, 3 and 5 share one packed head (head = 2); config 4
has its own (head = 4).  Config 1 is built from a dense head by the oracle's
constructor, so its stream instead draws Q0 -> calibration H -> h -> targets ->
the dense head W.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import numpy as np

SEED_BASE = 20260802


@dataclasses.dataclass(frozen=True)
class HeadShape:
    """Shape metadata of one packed head (the component list of §3.3)."""

    V: int      # vocabulary rows
    d: int      # hidden size
    r_c: int    # rank of the quantised core A_c B_c (Eq. 3)
    r_r: int    # rank of the activation-metric correction A_w B_w (Eq. 4-5)
    g: int      # group size of the signed-INT4 residual scales along d
    g_B: int    # group size of the INT8 correction factor B_w along d

    def as_tuple(self):
        return (self.V, self.d, self.r_c, self.r_r, self.g, self.g_B)


@dataclasses.dataclass(frozen=True)
class Workload:
    cfg: int
    name: str
    shape: HeadShape
    T: int                 # tokens per call
    head_seed_cfg: int     # which config's component stream the head comes from


# The five workloads.  Sizes follow the pages' head shapes (Qwen3-8B-Base
# 151,936 x 4,096; Gemma-4-E4B 262,144 x 2,560).
WORKLOADS: Dict[int, Workload] = {
    1: Workload(1, "tiny-built V1024 d256 T4", HeadShape(1024, 256, 32, 8, 64, 64), 4, 1),
    2: Workload(2, "qwen3-8b-head decode T1", HeadShape(151936, 4096, 512, 64, 128, 128), 1, 2),
    3: Workload(3, "qwen3-8b-head decode T64 sweep", HeadShape(151936, 4096, 512, 64, 128, 128), 64, 2),
    4: Workload(4, "gemma-4-e4b-head decode T16", HeadShape(262144, 2560, 384, 64, 128, 128), 16, 4),
    5: Workload(5, "qwen3-8b-head prefill T4096", HeadShape(151936, 4096, 512, 64, 128, 128), 4096, 2),
}
SWEEP_T = (2, 8, 32, 64)   # config 3 uses the first T rows of its 64-row draw

# The pages' storage-matched comparison heads at the Qwen3-8B shape, as shapes of
# the same packed format: a plain group-INT4 head (no low-rank branches) whose
# 16-column groups bring its bytes to ARCHead's, and the core + residual head
# without the metric correction.
BASELINE_SHAPES: Dict[str, HeadShape] = {
    "naive-int4": HeadShape(151936, 4096, 0, 0, 16, 128),
    "core-int4": HeadShape(151936, 4096, 512, 0, 128, 128),
}

# Scale magnitudes of the seeded components (standard deviations of the
# half-normal draws).  Each branch then contributes a comparable share of every
# head entry, so dropping any branch is visible.
SCALE_STD = dict(s_L=2e-3, s_R=1e-3, s_res=3e-3, s_A=2e-3, s_B=2.5e-4)


# ----------------------------------------------------------------- encodings
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """IEEE float32 -> bfloat16 bit pattern, round to nearest even (NaN kept quiet)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    r = ((u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)).astype(np.uint16)
    nan = np.isnan(np.asarray(x, dtype=np.float32))
    if nan.any():
        r = r.copy()
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def f64_to_fp16_bits(x: np.ndarray) -> np.ndarray:
    """IEEE binary16 bit pattern of x (numpy's float16 cast rounds to nearest even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)


# ------------------------------------------------------------------- draws
def _rng(seed_cfg: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(SEED_BASE + seed_cfg))


def anisotropic_basis(rng: np.random.Generator, d: int):
    """Random orthonormal basis Q0 (QR of a Gaussian with the sign fix) and the
    eigenvalue profile 10 * k^-1.5, k = 1..d."""
    G = rng.standard_normal((d, d))
    Q, Rm = np.linalg.qr(G)
    Q = Q * np.sign(np.diag(Rm))[None, :]
    lam = 10.0 * np.arange(1, d + 1, dtype=np.float64) ** -1.5
    return Q, lam


def anisotropic_rows(rng: np.random.Generator, Q: np.ndarray, lam: np.ndarray, n: int) -> np.ndarray:
    """n rows ~ N(0, Q diag(lam) Q^T), float64."""
    z = rng.standard_normal((n, Q.shape[0]))
    return (z * np.sqrt(lam)[None, :]) @ Q.T


def _half_normal_fp16(rng, std, shape):
    return f64_to_fp16_bits(np.abs(rng.standard_normal(shape)) * std)


def _codes(rng, lo, hi, shape):
    return rng.integers(lo, hi + 1, size=shape, dtype=np.int8)


def draw_components(shape: HeadShape, head_seed_cfg: int) -> Dict[str, np.ndarray]:
    """Seeded packed components in canonical form.

    Codes are int8 arrays holding two's-complement values in the format's range
    (INT5 [-16,15], INT8 [-128,127], INT4 [-8,7]); scales are fp16 bit patterns
    (uint16).
    """
    V, d, r_c, r_r, g, g_B = (shape.V, shape.d, shape.r_c, shape.r_r, shape.g, shape.g_B)
    rng = _rng(100 + head_seed_cfg)
    c: Dict[str, np.ndarray] = {}
    c["L"] = _codes(rng, -16, 15, (V, r_c))
    c["s_L"] = _half_normal_fp16(rng, SCALE_STD["s_L"], (V,))
    c["R"] = _codes(rng, -128, 127, (r_c, d))
    c["s_R"] = _half_normal_fp16(rng, SCALE_STD["s_R"], (r_c,))
    c["q"] = _codes(rng, -8, 7, (V, d))
    c["s_res"] = _half_normal_fp16(rng, SCALE_STD["s_res"], (V, d // g))
    c["A"] = _codes(rng, -128, 127, (V, r_r))
    c["s_A"] = _half_normal_fp16(rng, SCALE_STD["s_A"], (V,))
    c["B"] = _codes(rng, -128, 127, (r_r, d))
    c["s_B"] = _half_normal_fp16(rng, SCALE_STD["s_B"], (r_r, d // g_B))
    return c


def draw_activations(d: int, T: int, V: int, seed_cfg: int):
    """Hidden states h (bf16 bits, [T, d]) and target ids (int32, [T])."""
    rng = _rng(seed_cfg)
    Q, lam = anisotropic_basis(rng, d)
    h = anisotropic_rows(rng, Q, lam, T)
    h_bits = f32_to_bf16_bits(h.astype(np.float32))
    targets = rng.integers(0, V, size=T, dtype=np.int64).astype(np.int32)
    return h_bits, targets


def make_workload(cfg: int, T: Optional[int] = None, with_components: bool = True):
    """Inputs of workload ``cfg`` (2..5).  Returns (shape, h_bits, targets, comps).

    ``T`` overrides the token count (the activation draw then has that many rows).
    """
    wl = WORKLOADS[cfg]
    if cfg == 1:
        raise ValueError("config 1 is constructed from a dense head: use dense_head_inputs()")
    T = wl.T if T is None else T
    h_bits, targets = draw_activations(wl.shape.d, T, wl.shape.V, cfg)
    comps = draw_components(wl.shape, wl.head_seed_cfg) if with_components else None
    return wl.shape, h_bits, targets, comps


def dense_head_inputs(n_calib: int = 4096, T: int = 4, seed_cfg: int = 1, V: int = 1024, d: int = 256,
                      rank: int = 32, low_rank_std: float = 0.05, noise_std: float = 0.01):
    """Config 1 raw inputs: dense head W (float32 values held in float64),
    calibration states H (float64, [n_calib, d]), hidden states h (bf16 bits,
    [T, d]) and target ids.

    W = rank-``rank`` Gaussian part whose entries have std ``low_rank_std``
    plus i.i.d. Gaussian noise of std ``noise_std``.
    """
    rng = _rng(seed_cfg)
    Q, lam = anisotropic_basis(rng, d)
    H = anisotropic_rows(rng, Q, lam, n_calib)
    h = anisotropic_rows(rng, Q, lam, T)
    h_bits = f32_to_bf16_bits(h.astype(np.float32))
    targets = rng.integers(0, V, size=T, dtype=np.int64).astype(np.int32)
    G1 = rng.standard_normal((V, rank))
    G2 = rng.standard_normal((rank, d))
    W = low_rank_std * (G1 @ G2) / np.sqrt(rank) + noise_std * rng.standard_normal((V, d))
    W = W.astype(np.float32).astype(np.float64)
    return W, H, h_bits, targets


def dense_head_inputs_device(V: int, d: int, n_calib: int, seed: int = 11, rank: int = 32,
                             low_rank_std: float = 0.05, noise_std: float = 0.01, device: str = "cuda"):
    """Full-size dense head and calibration states drawn on the device (the
    config-1 recipe at any shape: W = rank-``rank`` Gaussian part + i.i.d.
    noise, H ~ N(0, Q0 diag(10 k^-1.5) Q0^T)), from a seeded torch generator.
    Returns fp32 tensors W [V, d] and H [n_calib, d]."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(SEED_BASE + seed)
    G1 = torch.randn(V, rank, device=device, generator=g, dtype=torch.float32)
    G2 = torch.randn(rank, d, device=device, generator=g, dtype=torch.float32)
    W = low_rank_std * (G1 @ G2) / math.sqrt(rank)
    W += noise_std * torch.randn(V, d, device=device, generator=g, dtype=torch.float32)
    Q, Rm = torch.linalg.qr(torch.randn(d, d, device=device, generator=g, dtype=torch.float64))
    Q = Q * torch.sign(torch.diagonal(Rm))[None, :]
    lam = 10.0 * torch.arange(1, d + 1, device=device, dtype=torch.float64) ** -1.5
    z = torch.randn(n_calib, d, device=device, generator=g, dtype=torch.float64)
    H = ((z * lam.sqrt()[None, :]) @ Q.T).float()
    return W, H


def random_components(shape: HeadShape, seed: int) -> Dict[str, np.ndarray]:
    """Small seeded components of an arbitrary shape (used for ragged and edge cases)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    V, d, r_c, r_r, g, g_B = (shape.V, shape.d, shape.r_c, shape.r_r, shape.g, shape.g_B)
    c: Dict[str, np.ndarray] = {}
    c["L"] = _codes(rng, -16, 15, (V, r_c))
    c["s_L"] = _half_normal_fp16(rng, SCALE_STD["s_L"], (V,))
    c["R"] = _codes(rng, -128, 127, (r_c, d))
    c["s_R"] = _half_normal_fp16(rng, SCALE_STD["s_R"], (r_c,))
    c["q"] = _codes(rng, -8, 7, (V, d))
    c["s_res"] = _half_normal_fp16(rng, SCALE_STD["s_res"], (V, d // g))
    c["A"] = _codes(rng, -128, 127, (V, r_r))
    c["s_A"] = _half_normal_fp16(rng, SCALE_STD["s_A"], (V,))
    c["B"] = _codes(rng, -128, 127, (r_r, d))
    c["s_B"] = _half_normal_fp16(rng, SCALE_STD["s_B"], (r_r, d // g_B))
    return c


def random_hidden(d: int, T: int, seed: int, V: int = 1):
    """Anisotropic bf16 hidden states for small edge-case shapes, plus targets."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Q, lam = anisotropic_basis(rng, d)
    h = anisotropic_rows(rng, Q, lam, T)
    targets = rng.integers(0, V, size=T, dtype=np.int64).astype(np.int32)
    return f32_to_bf16_bits(h.astype(np.float32)), targets
