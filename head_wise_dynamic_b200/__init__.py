"""Head-wise dynamic sparse global attention (SAF3R) for B200 (sm_100a).

Python binding of the C-ABI library `libsaf3r.so` (declared in include/saf3r.h).
This module only marshals arguments: every step of the path runs in the
library's CUDA kernels.  PyTorch supplies device memory and streams.  There is
no CPU fallback: importing works without a GPU, but every compute call needs
the compiled library and a B200.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# SAF3R_LIB may point at another build of the same library (e.g. a debug build).
LIB_PATH = os.environ.get("SAF3R_LIB") or os.path.join(_HERE, "libsaf3r.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "saf3r.h")

# saf3r_status
OK, ERR_INVALID, ERR_CUDA, ERR_TIMEOUT, ERR_INDEX, ERR_UNSUPPORTED = range(6)
# saf3r_head_type
POSITION, PROBE, CORR, SCAN, DENSE, HYBRID, TOKEN = range(7)
# workspace operations
OP_SELECT, OP_SPARSE, OP_DENSE, OP_PROFILE = range(4)


class Saf3rError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class saf3r_layout(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
                ("n_special", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
                ("dino_dim", ctypes.c_int32), ("tile", ctypes.c_int32)]


class saf3r_head_cfg(ctypes.Structure):
    _fields_ = [("type", ctypes.c_int32), ("k", ctypes.c_int32), ("stride", ctypes.c_int32),
                ("phase", ctypes.c_int32), ("radius", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C-ABI library (raises if it was never built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m head_wise_dynamic_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        LP, CP = ctypes.POINTER(saf3r_layout), ctypes.POINTER(saf3r_head_cfg)
        L.saf3r_cache_bytes.argtypes = [LP, CP]
        L.saf3r_cache_bytes.restype = sz
        L.saf3r_workspace_bytes.argtypes = [LP, CP, i32]
        L.saf3r_workspace_bytes.restype = sz
        L.saf3r_profile_workspace_bytes.argtypes = [LP, CP, i32]
        L.saf3r_profile_workspace_bytes.restype = sz
        L.saf3r_select_kv.argtypes = [LP, CP, vp, vp, vp, vp, vp, vp]
        L.saf3r_select_kv.restype = i32
        L.saf3r_sparse_attn.argtypes = [LP, CP, vp, vp, vp, vp, vp, i32, vp, vp]
        L.saf3r_sparse_attn.restype = i32
        L.saf3r_dense_attn.argtypes = [LP, vp, vp, vp, vp, i32, vp, vp]
        L.saf3r_dense_attn.restype = i32
        L.saf3r_profile_heads.argtypes = [LP, CP, i32, vp, vp, vp, vp, ctypes.c_double, CP,
                                          ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64), vp, vp]
        L.saf3r_profile_heads.restype = i32
        L.saf3r_cache_export.argtypes = [LP, CP, vp, i32, ctypes.POINTER(ctypes.c_int32), sz,
                                         ctypes.POINTER(ctypes.c_size_t), vp]
        L.saf3r_cache_export.restype = i32
        L.saf3r_kept_pairs.argtypes = [LP, CP, vp, ctypes.POINTER(ctypes.c_int64), vp]
        L.saf3r_kept_pairs.restype = i32
        L.saf3r_choose_eq2.argtypes = [i32, i32, i32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                                       i32, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_double)]
        L.saf3r_choose_eq2.restype = i32
        L.saf3r_set_kernel_events.argtypes = [vp, vp]
        L.saf3r_set_kernel_events.restype = None
        L.saf3r_set_wait_budget.argtypes = [ctypes.c_longlong]
        L.saf3r_set_wait_budget.restype = None
        L.saf3r_test_withhold_arrive.argtypes = []
        L.saf3r_test_withhold_arrive.restype = None
        L.saf3r_baseline_stride.argtypes = [ctypes.c_double]
        L.saf3r_baseline_stride.restype = ctypes.c_int32
        L.saf3r_check.argtypes = [vp]
        L.saf3r_check.restype = i32
        L.saf3r_last_launch_count.argtypes = []
        L.saf3r_last_launch_count.restype = i32
        L.saf3r_status_string.argtypes = [i32]
        L.saf3r_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().saf3r_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != OK:
        raise Saf3rError(status, where)


# ------------------------------------------------------------------ marshalling helpers

def make_layout(S: int, grid_h: int, grid_w: Optional[int] = None, H: int = 16, n_special: int = 5,
                d: int = 64, dino_dim: int = 384, tile: int = 64) -> saf3r_layout:
    return saf3r_layout(S, grid_h, grid_h if grid_w is None else grid_w, n_special, H, d, dino_dim, tile)


def layout_of(L) -> saf3r_layout:
    """Accept a saf3r_layout or any object with S, g (or grid_h/grid_w), H, n_special, d, dino_dim, tile."""
    if isinstance(L, saf3r_layout):
        return L
    gh = getattr(L, "grid_h", None) or getattr(L, "g")
    gw = getattr(L, "grid_w", None) or getattr(L, "g")
    return saf3r_layout(L.S, gh, gw, L.n_special, L.H, L.d, L.dino_dim, L.tile)


def cfg_array(heads: Sequence) -> ctypes.Array:
    """Per-head configs (objects with kind/type, k, stride, phase, radius) -> saf3r_head_cfg[H]."""
    arr = (saf3r_head_cfg * len(heads))()
    for i, h in enumerate(heads):
        kind = getattr(h, "kind", None)
        if kind is None:
            kind = getattr(h, "type")
        arr[i] = saf3r_head_cfg(int(kind), int(getattr(h, "k", 0)), int(getattr(h, "stride", 0)),
                                int(getattr(h, "phase", 0)), int(getattr(h, "radius", 1)))
    return arr


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ the C ABI, one call each

def saf3r_cache_bytes(layout, cfg) -> int:
    return int(lib().saf3r_cache_bytes(ctypes.byref(layout_of(layout)), _cfg(cfg)))


def saf3r_workspace_bytes(layout, cfg, op: int) -> int:
    return int(lib().saf3r_workspace_bytes(ctypes.byref(layout_of(layout)), _cfg(cfg), int(op)))


def saf3r_profile_workspace_bytes(layout, cand) -> int:
    c = _cfg(cand)
    return int(lib().saf3r_profile_workspace_bytes(ctypes.byref(layout_of(layout)), c, len(c)))


def _cfg(cfg):
    if cfg is None:
        return None
    if isinstance(cfg, ctypes.Array):
        return cfg
    return cfg_array(cfg)


def saf3r_select_kv(layout, cfg, q, k, dino, cache, workspace, stream=None):
    st = lib().saf3r_select_kv(ctypes.byref(layout_of(layout)), _cfg(cfg), _ptr(q), _ptr(k), _ptr(dino),
                               _ptr(cache), _ptr(workspace), _stream(stream))
    _check(st, "saf3r_select_kv")


def saf3r_select_kv_static(layout, cfg, q, k, dino, cache, stream=None):
    """saf3r_select_kv for callers that cannot allocate a device workspace: the scratch
    comes from a fixed 40 MiB array inside the library (see include/saf3r.h for the limit,
    the first-call set-up and the rule that overlapping calls race)."""
    f = lib().saf3r_select_kv_static
    f.argtypes = [ctypes.POINTER(saf3r_layout), ctypes.POINTER(saf3r_head_cfg)] + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    st = f(ctypes.byref(layout_of(layout)), _cfg(cfg), _ptr(q), _ptr(k), _ptr(dino), _ptr(cache), _stream(stream))
    _check(st, "saf3r_select_kv_static")


def saf3r_sparse_attn(layout, cfg, cache, q, k, v, out, workspace, stream=None, out_is_fp32: Optional[bool] = None):
    if out_is_fp32 is None:
        import torch
        out_is_fp32 = out.dtype == torch.float32
    st = lib().saf3r_sparse_attn(ctypes.byref(layout_of(layout)), _cfg(cfg), _ptr(cache), _ptr(q), _ptr(k),
                                 _ptr(v), _ptr(out), int(bool(out_is_fp32)), _ptr(workspace), _stream(stream))
    _check(st, "saf3r_sparse_attn")


def saf3r_dense_attn(layout, q, k, v, out, workspace, stream=None, out_is_fp32: Optional[bool] = None):
    if out_is_fp32 is None:
        import torch
        out_is_fp32 = out.dtype == torch.float32
    st = lib().saf3r_dense_attn(ctypes.byref(layout_of(layout)), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                int(bool(out_is_fp32)), _ptr(workspace), _stream(stream))
    _check(st, "saf3r_dense_attn")


def saf3r_profile_heads(layout, cand, q, k, v, dino, nmse_max, workspace, stream=None):
    """Returns (chosen cfg array [H], nmse [H][n_cand] float64, pairs [H][n_cand] int64)."""
    L = layout_of(layout)
    c = _cfg(cand)
    H = L.H
    chosen = (saf3r_head_cfg * H)()
    nmse = np.zeros((H, len(c)), dtype=np.float64)
    pairs = np.zeros((H, len(c)), dtype=np.int64)
    st = lib().saf3r_profile_heads(ctypes.byref(L), c, len(c), _ptr(q), _ptr(k), _ptr(v), _ptr(dino),
                                   float(nmse_max), chosen, nmse.ctypes.data_as(ctypes.POINTER(ctypes.c_double)),
                                   pairs.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _ptr(workspace),
                                   _stream(stream))
    _check(st, "saf3r_profile_heads")
    return chosen, nmse, pairs


def saf3r_choose_eq2(nmse, pairs, base: int):
    """The eq. 2 search (see include/saf3r.h) over per-input tables nmse [n_inputs][H][n_cand]
    and pairs [n_inputs][H][n_cand]; returns (choice int32 [H], mean nmse [H][n_cand])."""
    e = np.ascontiguousarray(nmse, dtype=np.float64)
    w = np.ascontiguousarray(pairs, dtype=np.int64)
    if e.ndim == 2:
        e, w = e[None], w[None]
    if e.ndim != 3 or e.shape != w.shape:
        raise ValueError("nmse and pairs must be [n_inputs][H][n_cand] tables of one shape")
    n_in, H, C = e.shape
    choice = np.zeros(H, dtype=np.int32)
    mean = np.zeros((H, C), dtype=np.float64)
    dp = ctypes.POINTER(ctypes.c_double)
    st = lib().saf3r_choose_eq2(n_in, H, C, e.ctypes.data_as(dp), w.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                                int(base), choice.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), mean.ctypes.data_as(dp))
    _check(st, "saf3r_choose_eq2")
    return choice, mean


def saf3r_baseline_stride(sigma: float) -> int:
    """Stride of the uniform-sampling baseline of sparsity at least sigma (the library's rule)."""
    s = int(lib().saf3r_baseline_stride(float(sigma)))
    if s < 1:
        raise ValueError("sigma must be in [0, 1)")
    return s


baseline_stride = saf3r_baseline_stride


def profile_heads_eq2(layout, cand, base: int, inputs, workspace, stream=None):
    """The eq. 2 search over a calibration set: saf3r_profile_heads on every input
    (q, k, v, dino), then saf3r_choose_eq2 over the per-input tables.
    Returns (choice int32 [H], mean nmse [H][n_cand], pairs [n_inputs][H][n_cand])."""
    tables, costs = [], []
    for q, k, v, dino in inputs:
        _, nmse, pairs = saf3r_profile_heads(layout, cand, q, k, v, dino, 0.0, workspace, stream)
        tables.append(nmse)
        costs.append(pairs)
    if not tables:
        raise ValueError("the calibration set is empty")
    choice, mean = saf3r_choose_eq2(np.stack(tables), np.stack(costs), base)
    return choice, mean, np.stack(costs)


def saf3r_cache_export(layout, cfg, cache, head: int, stream=None) -> np.ndarray:
    L = layout_of(layout)
    c = _cfg(cfg)
    n = ctypes.c_size_t(0)
    st = lib().saf3r_cache_export(ctypes.byref(L), c, _ptr(cache), int(head), None, 0, ctypes.byref(n),
                                  _stream(stream))
    _check(st, "saf3r_cache_export")
    out = np.zeros(n.value, dtype=np.int32)
    st = lib().saf3r_cache_export(ctypes.byref(L), c, _ptr(cache), int(head),
                                  out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), out.size, ctypes.byref(n),
                                  _stream(stream))
    _check(st, "saf3r_cache_export")
    return out


def saf3r_kept_pairs(layout, cfg, cache, stream=None) -> np.ndarray:
    L = layout_of(layout)
    out = np.zeros(L.H, dtype=np.int64)
    st = lib().saf3r_kept_pairs(ctypes.byref(L), _cfg(cfg), _ptr(cache),
                                out.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _stream(stream))
    _check(st, "saf3r_kept_pairs")
    return out


def saf3r_set_kernel_events(start=None, stop=None):
    """Record torch.cuda.Event pair around the attention kernel of following calls (None, None: off).

    torch creates CUDA events lazily: record each event once before handing it over."""
    lib().saf3r_set_kernel_events(None if start is None else start.cuda_event,
                                  None if stop is None else stop.cuda_event)


def saf3r_set_wait_budget(cycles: int = 0):
    """Budget (GPU clock cycles) of every bounded device wait of this thread's following calls; 0 = default."""
    lib().saf3r_set_wait_budget(int(cycles))


def saf3r_test_withhold_arrive():
    """Test hook: the next attention launch on this thread lets one pipeline wait run out (see saf3r.h)."""
    lib().saf3r_test_withhold_arrive()


def saf3r_check(stream=None):
    _check(lib().saf3r_check(_stream(stream)), "saf3r_check (device)")


def saf3r_last_launch_count() -> int:
    return int(lib().saf3r_last_launch_count())


# ------------------------------------------------------------------ convenience: buffers owned by torch

class SparseGlobalAttention:
    """One layer's worth of buffers for the select -> sparse-attention path.

    `select(q, k, dino)` builds the per-input index cache; `__call__(q, k, v)`
    runs sparse attention over it (any number of times, e.g. with fresh Q/K/V
    of later layer calls).  Cache, workspace and output live in torch device
    memory allocated here.
    """

    def __init__(self, layout, heads, device="cuda", out_dtype=None):
        import torch
        self.layout = layout_of(layout)
        self.cfg = cfg_array(heads)
        self.device = device
        self.out_dtype = out_dtype or torch.bfloat16
        cb = saf3r_cache_bytes(self.layout, self.cfg)
        if cb == 0:
            raise Saf3rError(ERR_INVALID, "invalid layout or head configuration")
        ws = max(saf3r_workspace_bytes(self.layout, self.cfg, OP_SELECT),
                 saf3r_workspace_bytes(self.layout, self.cfg, OP_SPARSE))
        self.cache = torch.empty(cb, dtype=torch.uint8, device=device)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device=device)
        L = self.layout
        N = L.S * (L.grid_h * L.grid_w + L.n_special)
        self.out = torch.empty((L.H, N, L.d), dtype=self.out_dtype, device=device)

    def select(self, q, k, dino=None, stream=None):
        saf3r_select_kv(self.layout, self.cfg, q, k, dino, self.cache, self.workspace, stream)

    def __call__(self, q, k, v, out=None, stream=None):
        out = self.out if out is None else out
        saf3r_sparse_attn(self.layout, self.cfg, self.cache, q, k, v, out, self.workspace, stream)
        return out


def header_functions() -> List[str]:
    """Names of the functions that include/saf3r.h declares."""
    import re
    txt = open(HEADER_PATH).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(saf3r_[a-z_0-9]+)\s*\(", txt)))
