"""ARCHead packed LM-head forward on B200 (sm_100a): Python binding.

This module only marshals arguments to the C ABI of ``libarchead.so``
(declared in ``include/archead.h``); every step of the forward pass runs in
the library's CUDA kernels.  PyTorch is used for device memory and streams.
There is no CPU path: importing this module without the built library raises.

Source method: "ARCHead: Activation-Metric Residual Correction for Large
Language Model Output Heads", §3.2 (Eq. 3, 6, 7) and §3.3 (packed layout).
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libarchead.so")
if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python quantized_output_head_b200/build.py`")
_lib = ctypes.CDLL(LIB_PATH)

ARCHEAD_OK, ARCHEAD_EINVAL, ARCHEAD_EALIGN, ARCHEAD_EUNSUP, ARCHEAD_ECUDA, ARCHEAD_ENOMEM, ARCHEAD_ETIMEOUT = (
    0, -1, -2, -3, -4, -5, -6)
STATUS_WAIT_TIMEOUT, STATUS_BAD_TARGET = 1, 2

EXPORTED = (
    "archead_packed_bytes", "archead_arena_bytes", "archead_pack_load", "archead_pack_image",
    "archead_workspace_bytes",
    "archead_logits", "archead_logits_lse_argmax", "archead_host_workspace_bytes", "archead_lse_argmax_host",
    "archead_workspace_status", "archead_set_profile_events", "archead_free", "archead_last_cuda_error",
    "archead_status_string", "archead_static_workspace_capacity", "archead_logits_lse_argmax_static",
    "archead_static_workspace_status", "archead_test_decode_waits", "archead_host_logits_workspace_bytes",
    "archead_logits_host",
    "archead_forward_kernel", "archead_set_vocab_shard", "archead_shard_partials", "archead_merge_shards",
    "archead_sample", "archead_sample_partials", "archead_merge_sample_shards",
)


class ArcheadDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("V", "d", "r_c", "r_r", "g", "g_B")]


class ArcheadHostComponents(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("L", "s_L", "R", "s_R", "q", "s_res", "A", "s_A", "B", "s_B")]


_vp, _sz, _i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
_sig = {
    "archead_packed_bytes": (_sz, [ctypes.POINTER(ArcheadDesc)]),
    "archead_arena_bytes": (_sz, [ctypes.POINTER(ArcheadDesc)]),
    "archead_pack_load": (ctypes.c_int, [ctypes.POINTER(ArcheadDesc), ctypes.POINTER(ArcheadHostComponents),
                                         _vp, _sz, _vp, ctypes.POINTER(_vp)]),
    "archead_pack_image": (ctypes.c_int, [ctypes.POINTER(ArcheadDesc), ctypes.POINTER(ArcheadHostComponents),
                                          _vp, _sz]),
    "archead_workspace_bytes": (_sz, [_vp, _i32]),
    "archead_host_workspace_bytes": (_sz, [_vp, _i32]),
    "archead_logits": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "archead_logits_lse_argmax": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "archead_lse_argmax_host": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "archead_host_logits_workspace_bytes": (_sz, [_vp, _i32]),
    "archead_logits_host": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "archead_workspace_status": (ctypes.c_int, [_vp, ctypes.c_int, _vp, ctypes.POINTER(ctypes.c_uint32)]),
    "archead_set_profile_events": (ctypes.c_int, [_vp, _vp, _vp]),
    "archead_static_workspace_capacity": (_sz, []),
    "archead_logits_lse_argmax_static": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _vp, _vp]),
    "archead_static_workspace_status": (ctypes.c_int, [ctypes.c_int, _vp, ctypes.POINTER(ctypes.c_uint32)]),
    "archead_forward_kernel": (ctypes.c_int, [_vp, _i32]),
    "archead_set_vocab_shard": (ctypes.c_int, [_vp, _i32, _i32]),
    "archead_sample": (ctypes.c_int, [_vp, _vp, _i32, ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64, _vp, _vp,
                                      _vp, _vp, _sz, _vp]),
    "archead_shard_partials": (ctypes.c_int, [_vp, _vp, _i32, _vp, _vp, _vp, _sz, _vp]),
    "archead_merge_shards": (ctypes.c_int, [_vp, _i32, _i32, _vp, _vp, _vp, _vp]),
    "archead_sample_partials": (ctypes.c_int, [_vp, _vp, _i32, ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64, _vp,
                                               _vp, _sz, _vp]),
    "archead_merge_sample_shards": (ctypes.c_int, [_vp, _i32, _i32, _vp, _vp]),
    "archead_test_decode_waits": (ctypes.c_int, [_vp, ctypes.c_uint64, ctypes.c_int]),
    "archead_free": (None, [_vp]),
    "archead_last_cuda_error": (ctypes.c_int, []),
    "archead_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}
for _name, (_res, _args) in _sig.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args


class ArcheadError(RuntimeError):
    def __init__(self, status: int, what: str):
        msg = _lib.archead_status_string(status).decode()
        if status == ARCHEAD_ECUDA:
            msg += f" (cudaError {_lib.archead_last_cuda_error()})"
        super().__init__(f"{what}: {msg} [{status}]")
        self.status = status


def _check(status: int, what: str) -> None:
    if status != ARCHEAD_OK:
        raise ArcheadError(status, what)


def _desc(V, d, r_c, r_r, g, g_B) -> ArcheadDesc:
    return ArcheadDesc(int(V), int(d), int(r_c), int(r_r), int(g), int(g_B))


def archead_packed_bytes(V, d, r_c, r_r, g, g_B) -> int:
    """Eq. 10 byte count of the packed head (0 if the shape is unsupported)."""
    return int(_lib.archead_packed_bytes(ctypes.byref(_desc(V, d, r_c, r_r, g, g_B))))


def archead_arena_bytes(V, d, r_c, r_r, g, g_B) -> int:
    return int(_lib.archead_arena_bytes(ctypes.byref(_desc(V, d, r_c, r_r, g, g_B))))


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


_COMPONENT_DTYPES = dict(L=np.int8, s_L=np.uint16, R=np.int8, s_R=np.uint16, q=np.int8, s_res=np.uint16,
                         A=np.int8, s_A=np.uint16, B=np.int8, s_B=np.uint16)


def archead_pack_image(V, d, r_c, r_r, g, g_B, comps: Dict[str, np.ndarray]) -> np.ndarray:
    """Host arena image (uint8) of a packed head, as archead_pack_load would copy it."""
    desc = _desc(V, d, r_c, r_r, g, g_B)
    n = int(_lib.archead_arena_bytes(ctypes.byref(desc)))
    if n == 0:
        raise ArcheadError(ARCHEAD_EUNSUP, "archead_arena_bytes")
    keep = {k: np.ascontiguousarray(comps[k], dtype=dt) for k, dt in _COMPONENT_DTYPES.items()}
    hc = ArcheadHostComponents(**{k: v.ctypes.data for k, v in keep.items()})
    img = np.empty(n, dtype=np.uint8)
    _check(_lib.archead_pack_image(ctypes.byref(desc), ctypes.byref(hc), img.ctypes.data, n), "archead_pack_image")
    return img


class PackedHead:
    """A packed head resident in a device arena, with its library handle.

    ``comps``: canonical components (codes as int8 arrays, scales as fp16 bit
    patterns in uint16 arrays), the state-dict list of §3.3.
    """

    def __init__(self, V, d, r_c, r_r, g, g_B, comps: Dict[str, np.ndarray], device: int = 0,
                 stream: Optional[torch.cuda.Stream] = None):
        self.shape = (int(V), int(d), int(r_c), int(r_r), int(g), int(g_B))
        self.V, self.d = int(V), int(d)
        self._desc = _desc(*self.shape)
        nbytes = int(_lib.archead_arena_bytes(ctypes.byref(self._desc)))
        if nbytes == 0:
            raise ArcheadError(ARCHEAD_EUNSUP, "archead_arena_bytes")
        self.device = torch.device("cuda", device)
        self.arena = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        self._keep = {k: np.ascontiguousarray(comps[k], dtype=dt) for k, dt in _COMPONENT_DTYPES.items()}
        hc = ArcheadHostComponents(**{k: v.ctypes.data for k, v in self._keep.items()})
        h = _vp()
        with torch.cuda.device(self.device):
            _check(_lib.archead_pack_load(ctypes.byref(self._desc), ctypes.byref(hc), self.arena.data_ptr(),
                                          nbytes, _stream_ptr(stream), ctypes.byref(h)), "archead_pack_load")
        self._keep = None
        self.handle = h
        self._ws: Dict[Tuple[str, int], torch.Tensor] = {}

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and h.value and _lib is not None:   # _lib is gone at interpreter exit
            _lib.archead_free(h)
            self.handle = None

    @property
    def packed_bytes(self) -> int:
        return int(_lib.archead_packed_bytes(ctypes.byref(self._desc)))

    def workspace_bytes(self, T: int) -> int:
        return int(_lib.archead_workspace_bytes(self.handle, int(T)))

    def workspace(self, T: int, host_form=False) -> torch.Tensor:
        """A zero-initialised workspace big enough for T tokens (cached per size).
        host_form: False (device calls), True (archead_lse_argmax_host) or
        "logits" (archead_logits_host)."""
        size = {False: _lib.archead_workspace_bytes, True: _lib.archead_host_workspace_bytes,
                "logits": _lib.archead_host_logits_workspace_bytes}[host_form]
        n = size(self.handle, int(T))
        if n == 0:
            raise ArcheadError(ARCHEAD_EINVAL, "workspace size")
        key = (str(host_form), n)
        ws = self._ws.get(key)
        if ws is None:
            ws = torch.zeros(n, dtype=torch.uint8, device=self.device)
            self._ws[key] = ws
        return ws

    # -------------------------------------------------------------- calls
    def logits_into(self, hidden: torch.Tensor, logits: Optional[torch.Tensor], argmax: Optional[torch.Tensor],
                    workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
        T = int(hidden.shape[0])
        _check(_lib.archead_logits(self.handle, hidden.data_ptr(), T, _ptr(logits), _ptr(argmax),
                                   workspace.data_ptr(), workspace.numel(), _stream_ptr(stream)), "archead_logits")

    def lse_argmax_into(self, hidden: torch.Tensor, targets: Optional[torch.Tensor], lse: torch.Tensor,
                        argmax: torch.Tensor, ce: Optional[torch.Tensor], workspace: torch.Tensor,
                        stream: Optional[torch.cuda.Stream] = None) -> None:
        T = int(hidden.shape[0])
        _check(_lib.archead_logits_lse_argmax(self.handle, hidden.data_ptr(), T, _ptr(targets), lse.data_ptr(),
                                              argmax.data_ptr(), _ptr(ce), workspace.data_ptr(),
                                              workspace.numel(), _stream_ptr(stream)),
               "archead_logits_lse_argmax")

    def logits(self, hidden: torch.Tensor, want_logits: bool = True, want_argmax: bool = True):
        """hidden: [T, d] bf16 (or its 16-bit patterns) on this device.  Returns (logits|None, argmax|None)."""
        _check_hidden(hidden, self.d)
        T = int(hidden.shape[0])
        lg = torch.empty((T, self.V), dtype=torch.float32, device=self.device) if want_logits else None
        am = torch.empty(T, dtype=torch.int32, device=self.device) if want_argmax else None
        self.logits_into(hidden, lg, am, self.workspace(T))
        return lg, am

    def lse_argmax(self, hidden: torch.Tensor, targets: Optional[torch.Tensor] = None):
        """Fused epilogue: returns (lse [T] fp32, argmax [T] int32, ce [T] fp32 | None)."""
        _check_hidden(hidden, self.d)
        T = int(hidden.shape[0])
        lse = torch.empty(T, dtype=torch.float32, device=self.device)
        am = torch.empty(T, dtype=torch.int32, device=self.device)
        ce = None
        if targets is not None:
            targets = targets.to(device=self.device, dtype=torch.int32).contiguous()
            ce = torch.empty(T, dtype=torch.float32, device=self.device)
        self.lse_argmax_into(hidden, targets, lse, am, ce, self.workspace(T))
        return lse, am, ce

    def lse_argmax_host(self, hidden_host: np.ndarray, targets_host: Optional[np.ndarray] = None,
                        out: Optional[Tuple[np.ndarray, np.ndarray, Optional[np.ndarray]]] = None,
                        stream: Optional[torch.cuda.Stream] = None):
        """Host-buffer form: numpy (ideally pinned) in, numpy out; synchronises the stream."""
        hb = np.ascontiguousarray(hidden_host).view(np.uint16)
        T = int(hb.shape[0])
        tg = None if targets_host is None else np.ascontiguousarray(targets_host, dtype=np.int32)
        if out is None:
            out = (np.empty(T, np.float32), np.empty(T, np.int32), None if tg is None else np.empty(T, np.float32))
        lse, am, ce = out
        ws = self.workspace(T, host_form=True)
        _check(_lib.archead_lse_argmax_host(self.handle, hb.ctypes.data, T, None if tg is None else tg.ctypes.data,
                                            lse.ctypes.data, am.ctypes.data, None if ce is None else ce.ctypes.data,
                                            ws.data_ptr(), ws.numel(), _stream_ptr(stream)),
               "archead_lse_argmax_host")
        return lse, am, ce

    def logits_host(self, hidden_host: np.ndarray,
                    out: Optional[Tuple[Optional[np.ndarray], Optional[np.ndarray]]] = None,
                    stream: Optional[torch.cuda.Stream] = None):
        """Host-buffer logits: numpy bf16 bits [T, d] (ideally pinned) in,
        (logits [T, V] fp32, argmax [T] int32) numpy out; synchronises the stream."""
        hb = np.ascontiguousarray(hidden_host).view(np.uint16)
        T = int(hb.shape[0])
        if out is None:
            out = (np.empty((T, self.V), np.float32), np.empty(T, np.int32))
        lg, am = out
        ws = self.workspace(T, host_form="logits")
        _check(_lib.archead_logits_host(self.handle, hb.ctypes.data, T, None if lg is None else lg.ctypes.data,
                                        None if am is None else am.ctypes.data, ws.data_ptr(), ws.numel(),
                                        _stream_ptr(stream)), "archead_logits_host")
        return lg, am

    def prepare_logits_host(self, hidden_host: np.ndarray, out: Tuple[Optional[np.ndarray], Optional[np.ndarray]],
                            stream: Optional[torch.cuda.Stream] = None):
        """archead_logits_host bound to fixed host buffers (pinned memory lets
        the library replay one captured launch sequence): returns a callable
        that runs the call again on the current contents of those buffers.
        The buffers, the workspace and the stream are resolved once here."""
        hb = np.ascontiguousarray(hidden_host).view(np.uint16)
        T = int(hb.shape[0])
        lg, am = out
        ws = self.workspace(T, host_form="logits")
        args = (self.handle, hb.ctypes.data, T, None if lg is None else lg.ctypes.data,
                None if am is None else am.ctypes.data, ws.data_ptr(), ws.numel(), _stream_ptr(stream))
        return _bound_call(_lib.archead_logits_host, args, (hb, lg, am, ws), "archead_logits_host")

    def prepare_lse_argmax_host(self, hidden_host: np.ndarray, targets_host: Optional[np.ndarray],
                                out: Tuple[np.ndarray, np.ndarray, Optional[np.ndarray]],
                                stream: Optional[torch.cuda.Stream] = None):
        """archead_lse_argmax_host bound to fixed host buffers; see prepare_logits_host."""
        hb = np.ascontiguousarray(hidden_host).view(np.uint16)
        T = int(hb.shape[0])
        tg = None if targets_host is None else np.ascontiguousarray(targets_host, dtype=np.int32)
        lse, am, ce = out
        ws = self.workspace(T, host_form=True)
        args = (self.handle, hb.ctypes.data, T, None if tg is None else tg.ctypes.data, lse.ctypes.data,
                am.ctypes.data, None if ce is None else ce.ctypes.data, ws.data_ptr(), ws.numel(), _stream_ptr(stream))
        return _bound_call(_lib.archead_lse_argmax_host, args, (hb, tg, lse, am, ce, ws), "archead_lse_argmax_host")

    def sample(self, hidden: torch.Tensor, temperature: float, seed: int, offset: int = 0):
        """Gumbel-max temperature sampling fused into the vocabulary pass: returns
        (sampled [T] int32, lse [T], argmax [T]) of this head's rows; token t
        draws its noise at Philox counter offset + t under key seed."""
        _check_hidden(hidden, self.d)
        T = int(hidden.shape[0])
        out = torch.empty(T, dtype=torch.int32, device=self.device)
        lse = torch.empty(T, dtype=torch.float32, device=self.device)
        am = torch.empty(T, dtype=torch.int32, device=self.device)
        ws = self.workspace(T)
        _check(_lib.archead_sample(self.handle, hidden.data_ptr(), T, float(temperature), int(seed), int(offset),
                                   out.data_ptr(), lse.data_ptr(), am.data_ptr(), ws.data_ptr(), ws.numel(),
                                   _stream_ptr(None)), "archead_sample")
        return out, lse, am

    # --------------------------------------------------- vocabulary shards
    def set_vocab_shard(self, row_offset: int, vocab_total: int) -> None:
        """This head holds global rows [row_offset, row_offset + V) of a
        vocabulary of vocab_total rows: argmax and target ids become global."""
        _check(_lib.archead_set_vocab_shard(self.handle, int(row_offset), int(vocab_total)),
               "archead_set_vocab_shard")
        self.row_offset, self.vocab_total = int(row_offset), int(vocab_total)

    def shard_partials(self, hidden: torch.Tensor, targets: Optional[torch.Tensor] = None) -> torch.Tensor:
        """Per-token softmax statistics of this shard: [T, 4] fp32 rows
        (lse over the shard's rows, max logit, global argmax as int32 bits,
        target logit or NaN)."""
        _check_hidden(hidden, self.d)
        T = int(hidden.shape[0])
        if targets is not None:
            targets = targets.to(device=self.device, dtype=torch.int32).contiguous()
        out = torch.empty((T, 4), dtype=torch.float32, device=self.device)
        ws = self.workspace(T)
        _check(_lib.archead_shard_partials(self.handle, hidden.data_ptr(), T, _ptr(targets), out.data_ptr(),
                                           ws.data_ptr(), ws.numel(), _stream_ptr(None)), "archead_shard_partials")
        return out

    def sample_partials(self, hidden: torch.Tensor, temperature: float, seed: int, offset: int = 0) -> torch.Tensor:
        """This shard's share of a sampled draw: [T, 2] fp32 rows (the largest
        y / temperature + G over its rows, the global row as int32 bits), the
        noise of each global row as sample() draws it."""
        _check_hidden(hidden, self.d)
        T = int(hidden.shape[0])
        out = torch.empty((T, 2), dtype=torch.float32, device=self.device)
        ws = self.workspace(T)
        _check(_lib.archead_sample_partials(self.handle, hidden.data_ptr(), T, float(temperature), int(seed),
                                            int(offset), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream_ptr(None)),
               "archead_sample_partials")
        return out

    def forward_kernel(self, T: int) -> str:
        """'decode' or 'tensor_core': the kernel a call with T tokens runs on."""
        k = _lib.archead_forward_kernel(self.handle, int(T))
        if k < 0:
            raise ArcheadError(ARCHEAD_EINVAL, "archead_forward_kernel")
        return "tensor_core" if k == 1 else "decode"

    def set_profile_events(self, before, after) -> None:
        """Record `before` / `after` (cudaEvent_t handles as ints, or objects with a
        ``cuda_event`` attribute) around the vocabulary pass of every later call.
        None, None switches it off."""
        def raw(e):
            return None if e is None else int(getattr(e, "cuda_event", e))
        b, a = raw(before), raw(after)
        _check(_lib.archead_set_profile_events(self.handle, b, a), "archead_set_profile_events")

    def status(self, workspace: torch.Tensor, clear: bool = True) -> int:
        v = ctypes.c_uint32(0)
        rc = _lib.archead_workspace_status(workspace.data_ptr(), 1 if clear else 0, _stream_ptr(None),
                                           ctypes.byref(v))
        if rc not in (ARCHEAD_OK, ARCHEAD_ETIMEOUT):
            _check(rc, "archead_workspace_status")
        return int(v.value)


def _bound_call(fn, args, keep, what):
    """A no-argument call of `fn(*args)` that raises on a non-OK status; `keep`
    holds the buffers the arguments point into."""
    def call():
        rc = fn(*args)
        if rc != ARCHEAD_OK:
            raise ArcheadError(rc, what)
    call.buffers = keep
    return call


# ------------------------------------------------------- vocabulary shards
def shard_rows(V: int, world: int, rank: int, tile: int = 128) -> Tuple[int, int]:
    """Rows [v0, v1) of rank `rank` among `world` vocabulary shards: whole
    128-row tiles split as evenly as possible, in rank order."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    tiles = -(-V // tile)
    t0 = rank * tiles // world
    t1 = (rank + 1) * tiles // world
    return min(V, t0 * tile), min(V, t1 * tile)


# Components indexed by vocabulary row (the rest, R, B and their scales, are
# shared by every shard).
_ROW_COMPONENTS = ("L", "s_L", "q", "s_res", "A", "s_A")


def shard_components(comps: Dict[str, np.ndarray], v0: int, v1: int) -> Dict[str, np.ndarray]:
    """The canonical components of rows [v0, v1) of a head."""
    return {k: (np.ascontiguousarray(v[v0:v1]) if k in _ROW_COMPONENTS else v) for k, v in comps.items()}


def gather_partials(parts: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather every rank's shard partials ([T, 4] statistics or [T, 2]
    sampling pairs) into [world, T, ...], in rank order (the one cross-GPU
    exchange of a vocabulary-sharded head)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    bufs = [torch.empty_like(parts) for _ in range(world)]
    dist.all_gather(bufs, parts.contiguous(), group=group)
    return torch.stack(bufs)


def merge_shards(parts: torch.Tensor):
    """Fold [n_shards, T, 4] partials (increasing row order) into
    (lse [T], argmax [T] int32, ce [T]); all on the partials' CUDA device."""
    if parts.dim() != 3 or parts.shape[2] != 4 or parts.dtype != torch.float32 or not parts.is_cuda:
        raise ValueError("parts must be a [n_shards, T, 4] float32 CUDA tensor")
    parts = parts.contiguous()
    n, T = int(parts.shape[0]), int(parts.shape[1])
    lse = torch.empty(T, dtype=torch.float32, device=parts.device)
    am = torch.empty(T, dtype=torch.int32, device=parts.device)
    ce = torch.empty(T, dtype=torch.float32, device=parts.device)
    with torch.cuda.device(parts.device):
        _check(_lib.archead_merge_shards(parts.data_ptr(), n, T, lse.data_ptr(), am.data_ptr(), ce.data_ptr(),
                                         _stream_ptr(None)), "archead_merge_shards")
    return lse, am, ce


def merge_sample_shards(parts: torch.Tensor) -> torch.Tensor:
    """Fold [n_shards, T, 2] sampling pairs (increasing row order) into the
    sampled ids [T] int32: the draw of the unsharded head."""
    if parts.dim() != 3 or parts.shape[2] != 2 or parts.dtype != torch.float32 or not parts.is_cuda:
        raise ValueError("parts must be a [n_shards, T, 2] float32 CUDA tensor")
    parts = parts.contiguous()
    n, T = int(parts.shape[0]), int(parts.shape[1])
    out = torch.empty(T, dtype=torch.int32, device=parts.device)
    with torch.cuda.device(parts.device):
        _check(_lib.archead_merge_sample_shards(parts.data_ptr(), n, T, out.data_ptr(), _stream_ptr(None)),
               "archead_merge_sample_shards")
    return out


def _check_hidden(hidden: torch.Tensor, d: int) -> None:
    if hidden.dim() != 2 or hidden.shape[1] != d or hidden.element_size() != 2 or not hidden.is_contiguous():
        raise ValueError(f"hidden must be a contiguous [T, {d}] tensor of 16-bit (bf16) elements")
    if not hidden.is_cuda:
        raise ValueError("hidden must be on the CUDA device")
