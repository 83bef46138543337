"""GPU construction of an ARCHead packed head: Python binding of
``libarchead_build.so`` (declared in ``include/archead_build.h``).

Argument marshalling only: the metric, the truncated SVDs, the quantisers and
the residuals all run in the library (its kernels, cuBLAS and cuSOLVER), in
fp64.  PyTorch supplies device memory and the stream.  Importing this module
without the built library raises.

Source method: "ARCHead: Activation-Metric Residual Correction for Large
Language Model Output Heads", §3.1 (Eq. 1-2), §3.2 (Eq. 3-5) and Algorithm 1
(§3.4).
"""
from __future__ import annotations

import ctypes
import importlib.util
import os
from typing import Dict, Tuple

import numpy as np
import torch

from . import ArcheadDesc

_PKG = os.path.dirname(os.path.abspath(__file__))
BUILD_LIB_PATH = os.path.join(_PKG, "libarchead_build.so")
if not os.path.exists(BUILD_LIB_PATH):
    raise ImportError(f"{BUILD_LIB_PATH} is not built; run `python quantized_output_head_b200/build.py`")


def _preload_cuda_libraries() -> None:
    """Load cuBLAS / cuSOLVER (and what cuSOLVER needs) from the nvidia wheels
    PyTorch uses, so the builder shares PyTorch's copies instead of mixing in
    another toolkit's from the loader path."""
    order = (("nvidia.cublas", "libcublasLt.so.12"), ("nvidia.cublas", "libcublas.so.12"),
             ("nvidia.nvjitlink", "libnvJitLink.so.12"), ("nvidia.cusparse", "libcusparse.so.12"),
             ("nvidia.cusolver", "libcusolver.so.11"))
    for mod, name in order:
        try:
            spec = importlib.util.find_spec(mod)
        except ImportError:
            spec = None
        if spec is None or not spec.submodule_search_locations:
            continue
        path = os.path.join(list(spec.submodule_search_locations)[0], "lib", name)
        if os.path.exists(path):
            ctypes.CDLL(path, mode=ctypes.RTLD_GLOBAL)


_preload_cuda_libraries()
_blib = ctypes.CDLL(BUILD_LIB_PATH)

EXPORTED_BUILD = (
    "archead_build_workspace_bytes", "archead_build_quantize", "archead_build_metric",
    "archead_build_correction", "archead_build_head", "archead_build_correction_svd", "archead_build_head_svd",
    "archead_build_last_error",
)
ARCHEAD_SVD_EXACT, ARCHEAD_SVD_RANDOMIZED = 0, 1
# Defaults of the randomised truncated SVD (sketch columns r + oversample,
# subspace iteration steps); see archead_svd_opts.
RANDOMIZED_OVERSAMPLE, RANDOMIZED_POWER_ITERS = 32, 2


class ArcheadSvdOpts(ctypes.Structure):
    _fields_ = [("method", ctypes.c_int32), ("oversample", ctypes.c_int32), ("power_iters", ctypes.c_int32),
                ("seed", ctypes.c_uint64)]


class ArcheadDeviceComponents(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("L", "s_L", "R", "s_R", "q", "s_res", "A", "s_A", "B", "s_B")]


_vp, _sz, _i32, _f64 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_double
_DESC = ctypes.POINTER(ArcheadDesc)
_sig = {
    "archead_build_workspace_bytes": (_sz, [_DESC, _i32]),
    "archead_build_quantize": (ctypes.c_int, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "archead_build_metric": (ctypes.c_int, [_i32, _i32, _vp, _f64, _f64, _vp, _vp, _vp, _sz, _vp]),
    "archead_build_correction": (ctypes.c_int, [_DESC, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "archead_build_head": (ctypes.c_int, [_DESC, _vp, _vp, _i32, _f64, _f64, ctypes.POINTER(ArcheadDeviceComponents),
                                          _vp, _sz, _vp]),
    "archead_build_correction_svd": (ctypes.c_int, [_DESC, _vp, _vp, _vp, ctypes.POINTER(ArcheadSvdOpts), _vp, _vp,
                                                    _vp, _vp, _vp, _sz, _vp]),
    "archead_build_head_svd": (ctypes.c_int, [_DESC, _vp, _vp, _i32, _f64, _f64, ctypes.POINTER(ArcheadSvdOpts),
                                              ctypes.POINTER(ArcheadDeviceComponents), _vp, _sz, _vp]),
    "archead_build_last_error": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_blib, _name)
    _f.restype = _res
    _f.argtypes = _args


class ArcheadBuildError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: status {status}: {_blib.archead_build_last_error().decode()}")
        self.status = status


def _check(status: int, what: str) -> None:
    if status != 0:
        raise ArcheadBuildError(status, what)


def _stream() -> int:
    return int(torch.cuda.current_stream().cuda_stream)


def _dev(t: torch.Tensor, dtype: torch.dtype, name: str) -> torch.Tensor:
    if not (t.is_cuda and t.dtype == dtype and t.is_contiguous()):
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    return t


def _desc(V, d, r_c, r_r, g, g_B) -> ArcheadDesc:
    return ArcheadDesc(int(V), int(d), int(r_c), int(r_r), int(g), int(g_B))


def workspace(V, d, r_c, r_r, g, g_B, n_calib: int) -> torch.Tensor:
    n = int(_blib.archead_build_workspace_bytes(ctypes.byref(_desc(V, d, r_c, r_r, g, g_B)), int(n_calib)))
    if n == 0:
        raise ArcheadBuildError(-1, "archead_build_workspace_bytes")
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def quantize(x: torch.Tensor, bits: int, group: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """Symmetric quantiser of §3.2 on a [rows, cols] fp64 CUDA tensor: codes
    (int8) and fp16 scale bits (int16 storage, [rows, cols / group]); group 0
    = one scale per row."""
    _dev(x, torch.float64, "x")
    rows, cols = x.shape
    G = cols if group == 0 else int(group)
    codes = torch.empty(rows, cols, dtype=torch.int8, device=x.device)
    scales = torch.empty(rows, cols // G if G and cols % G == 0 else 1, dtype=torch.int16, device=x.device)
    _check(_blib.archead_build_quantize(x.data_ptr(), rows, cols, int(bits), int(group), codes.data_ptr(),
                                        scales.data_ptr(), _stream()), "archead_build_quantize")
    return codes, scales


def metric(H: torch.Tensor, lam: float, p: float) -> Tuple[torch.Tensor, torch.Tensor]:
    """Eq. 1-2: (T_p, T_p^-1), fp64 [d, d], from calibration states H [N, d] (fp32)."""
    _dev(H, torch.float32, "H")
    N, d = H.shape
    ws = workspace(1, d, 0, 0, 1, 1, N)
    T_p = torch.empty(d, d, dtype=torch.float64, device=H.device)
    T_inv = torch.empty_like(T_p)
    _check(_blib.archead_build_metric(d, N, H.data_ptr(), float(lam), float(p), T_p.data_ptr(), T_inv.data_ptr(),
                                      ws.data_ptr(), ws.numel(), _stream()), "archead_build_metric")
    return T_p, T_inv


def svd_opts(svd: str = "exact", oversample: int = RANDOMIZED_OVERSAMPLE, power_iters: int = RANDOMIZED_POWER_ITERS,
             seed: int = 0) -> ArcheadSvdOpts:
    """archead_svd_opts for svd = "exact" or "randomized"."""
    if svd not in ("exact", "randomized"):
        raise ValueError(f"svd must be 'exact' or 'randomized', not {svd!r}")
    method = ARCHEAD_SVD_EXACT if svd == "exact" else ARCHEAD_SVD_RANDOMIZED
    return ArcheadSvdOpts(method, int(oversample), int(power_iters), int(seed) & (2**64 - 1))


def correction(E: torch.Tensor, T_p: torch.Tensor, T_inv: torch.Tensor, r_r: int, g_B: int, svd: str = "exact",
               **svd_kw) -> Dict[str, torch.Tensor]:
    """Eq. 4-5 with INT8 factors: A, s_A, B, s_B from the core's remainder E [V, d]
    (svd: "exact" or "randomized", with svd_opts' keywords)."""
    for t, n in ((E, "E"), (T_p, "T_p"), (T_inv, "T_inv")):
        _dev(t, torch.float64, n)
    V, d = E.shape
    desc = _desc(V, d, 0, r_r, 1, g_B)
    ws = workspace(V, d, 0, r_r, 1, g_B, 1)
    out = dict(A=torch.empty(V, r_r, dtype=torch.int8, device=E.device),
               s_A=torch.empty(V, dtype=torch.int16, device=E.device),
               B=torch.empty(r_r, d, dtype=torch.int8, device=E.device),
               s_B=torch.empty(r_r, d // g_B, dtype=torch.int16, device=E.device))
    opts = svd_opts(svd, **svd_kw)
    _check(_blib.archead_build_correction_svd(ctypes.byref(desc), E.data_ptr(), T_p.data_ptr(), T_inv.data_ptr(),
                                              ctypes.byref(opts), out["A"].data_ptr(), out["s_A"].data_ptr(),
                                              out["B"].data_ptr(), out["s_B"].data_ptr(), ws.data_ptr(), ws.numel(),
                                              _stream()),
           "archead_build_correction_svd")
    return out


def build_head(W: torch.Tensor, H: torch.Tensor, r_c: int, r_r: int, g: int, g_B: int, p: float = 0.75,
               lam: float = 1e-2, ws: torch.Tensor = None, svd: str = "exact", **svd_kw) -> Dict[str, torch.Tensor]:
    """Algorithm 1: every packed component (device tensors, canonical names;
    scales as int16 storage of fp16 bits) from the dense head W [V, d] and
    calibration states H [N, d], both fp32 CUDA tensors.  svd: "exact" or
    "randomized" (the truncated SVDs; svd_opts' keywords)."""
    _dev(W, torch.float32, "W")
    _dev(H, torch.float32, "H")
    V, d = W.shape
    N = H.shape[0]
    if H.shape[1] != d:
        raise ValueError("H and W disagree on d")
    desc = _desc(V, d, r_c, r_r, g, g_B)
    if ws is None:
        ws = workspace(V, d, r_c, r_r, g, g_B, N)
    dev = W.device
    out = dict(L=torch.empty(V, r_c, dtype=torch.int8, device=dev), s_L=torch.empty(V, dtype=torch.int16, device=dev),
               R=torch.empty(r_c, d, dtype=torch.int8, device=dev), s_R=torch.empty(r_c, dtype=torch.int16, device=dev),
               q=torch.empty(V, d, dtype=torch.int8, device=dev),
               s_res=torch.empty(V, d // g, dtype=torch.int16, device=dev),
               A=torch.empty(V, r_r, dtype=torch.int8, device=dev), s_A=torch.empty(V, dtype=torch.int16, device=dev),
               B=torch.empty(r_r, d, dtype=torch.int8, device=dev),
               s_B=torch.empty(r_r, d // g_B, dtype=torch.int16, device=dev))
    dc = ArcheadDeviceComponents(**{k: (v.data_ptr() if v.numel() else None) for k, v in out.items()})
    opts = svd_opts(svd, **svd_kw)
    _check(_blib.archead_build_head_svd(ctypes.byref(desc), W.data_ptr(), H.data_ptr(), N, float(lam), float(p),
                                        ctypes.byref(opts), ctypes.byref(dc), ws.data_ptr(), ws.numel(), _stream()),
           "archead_build_head_svd")
    return out


def to_host(comps: Dict[str, torch.Tensor]) -> Dict[str, np.ndarray]:
    """Device components -> the host dict PackedHead takes (int8 codes, uint16 scale bits)."""
    host = {}
    for k, v in comps.items():
        a = v.cpu().numpy()
        host[k] = a.view(np.uint16) if a.dtype == np.int16 else a
    return host
