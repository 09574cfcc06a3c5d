"""Thin ctypes binding of libug (include/ug.h): argument marshalling only.

Every function keeps the C name.  Tensors are torch tensors (device memory
and streams come from PyTorch); every step of the layer runs in the
library's CUDA kernels.  If libug.so is missing the first call raises; there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libug.so")
# The same library built with -DUG_DEBUG=1: a range check before every global
# access whose index a kernel computes (failures reach ug_check_error).
LIB_DEBUG_PATH = os.path.join(_HERE, "libug_debug.so")

UG_OK = 0
UG_ERR_INVALID_ARG = 1
UG_ERR_UNSUPPORTED = 2
UG_ERR_ALIGNMENT = 3
UG_ERR_ALIAS = 4
UG_ERR_CUDA = 5
UG_ERR_TIMEOUT = 6
UG_ERR_NO_MEMORY = 7

UG_HR_WINDOW_FIRST = 0
UG_HR_RASTER = 1
UG_LR = 2

# Every symbol include/ug.h declares.
EXPORTS = (
    "ug_geom_validate", "ug_index_map_sizes", "ug_build_index_maps", "ug_visible_pairs",
    "ug_work_list_sizes", "ug_build_work_lists",
    "ug_status_string", "ug_plan_create", "ug_plan_destroy", "ug_get_index_maps",
    "ug_permute_window_first", "ug_permute_rope_window_first", "ug_unpermute", "ug_rope_2d",
    "ug_hier_local_attn_fwd", "ug_hier_local_attn_fwd_vo_raster",
    "ug_layer_workspace_bytes", "ug_layer_fwd", "ug_layer_fwd_static_scratch",
    "ug_plan_set_wait_timeout", "ug_check_error", "ug_warm_start", "ug_warm_start_stencil_weights",
    "ug_rope_2d_bwd", "ug_unpermute_rope_bwd", "ug_attn_bwd_workspace_bytes",
    "ug_hier_local_attn_bwd", "ug_hier_local_attn_bwd_vo_raster",
    "ug_layer_bwd_workspace_bytes", "ug_layer_bwd",
)

# Capacity of the static scratch of ug_layer_fwd_static_scratch (ug.h).
UG_STATIC_SCRATCH_BYTES = 32 << 20


class UgError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


class ug_geom(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("grid_h", ctypes.c_int32), ("grid_w", ctypes.c_int32),
        ("win_h", ctypes.c_int32), ("win_w", ctypes.c_int32), ("radius", ctypes.c_int32),
        ("lr_h", ctypes.c_int32), ("lr_w", ctypes.c_int32), ("rho", ctypes.c_double),
        ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
        ("rope_dim_y", ctypes.c_int32), ("rope_dim_x", ctypes.c_int32),
        ("rope_theta", ctypes.c_double), ("softmax_scale", ctypes.c_float),
        ("text_len", ctypes.c_int32),
    ]


class ug_warm_start_params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("channels", ctypes.c_int32), ("lr_h", ctypes.c_int32),
        ("lr_w", ctypes.c_int32), ("scale", ctypes.c_int32), ("sharpen", ctypes.c_float),
        ("t", ctypes.c_float),
    ]


_lib = None
_loaded = {}


def lib() -> ctypes.CDLL:
    """The library the binding currently uses (LIB_PATH unless use_library
    chose another); loaded once per path, raises if it was not built."""
    global _lib
    if _lib is not None:
        return _lib
    _lib = _load(LIB_PATH)
    return _lib


def use_library(path: str) -> ctypes.CDLL:
    """Makes the library at path (e.g. LIB_DEBUG_PATH) the one that new plans
    and module-level calls use; plans already created keep theirs.  Returns
    the library that was in use before."""
    global _lib
    prev = lib()
    _lib = _load(path)
    return prev


def _set_library(L: ctypes.CDLL) -> None:
    global _lib
    _lib = L


def _load(path: str) -> ctypes.CDLL:
    if path in _loaded:
        return _loaded[path]
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m block_sparse_local_raster_b200.build`")
    L = ctypes.CDLL(path)
    P, I32, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    G = ctypes.POINTER(ug_geom)
    pi32 = ctypes.POINTER(ctypes.c_int32)
    pi64 = ctypes.POINTER(ctypes.c_int64)
    sig = {
        "ug_geom_validate": (I32, [G]),
        "ug_index_map_sizes": (I32, [G, pi64, pi64, pi64]),
        "ug_build_index_maps": (I32, [G, pi32, pi32, pi32]),
        "ug_visible_pairs": (I32, [G, pi64, pi64, pi64]),
        "ug_work_list_sizes": (I32, [G, pi64, pi64, pi64, pi64]),
        "ug_build_work_lists": (I32, [G, pi32, ctypes.POINTER(ctypes.c_uint32), pi32,
                                      ctypes.POINTER(ctypes.c_uint32)]),
        "ug_status_string": (ctypes.c_char_p, [I32]),
        "ug_plan_create": (I32, [G, ctypes.POINTER(P)]),
        "ug_plan_destroy": (I32, [P]),
        "ug_get_index_maps": (I32, [P, pi32, pi32, pi32]),
        "ug_permute_window_first": (I32, [P, P, P, P]),
        "ug_permute_rope_window_first": (I32, [P, P, P, P]),
        "ug_unpermute": (I32, [P, P, P, P]),
        "ug_rope_2d": (I32, [P, P, P, I32, P]),
        "ug_hier_local_attn_fwd": (I32, [P, P, P, P, P, P, P, P, P, P, P]),
        "ug_hier_local_attn_fwd_vo_raster": (I32, [P, P, P, P, P, P, P, P, P, P, P]),
        "ug_layer_workspace_bytes": (I64, [P]),
        "ug_layer_fwd": (I32, [P, P, P, P, P, P, P, P, P, P, P, I64, P]),
        "ug_layer_fwd_static_scratch": (I32, [P, P, P, P, P, P, P, P, P, P, P]),
        "ug_plan_set_wait_timeout": (I32, [P, I64]),
        "ug_check_error": (I32, [P, P]),
        "ug_warm_start": (I32, [ctypes.POINTER(ug_warm_start_params), P, P, P, P]),
        "ug_warm_start_stencil_weights": (I32, [ctypes.c_float, ctypes.c_float,
                                                ctypes.POINTER(ctypes.c_float)]),
        "ug_rope_2d_bwd": (I32, [P, P, P, I32, P]),
        "ug_unpermute_rope_bwd": (I32, [P, P, P, P]),
        "ug_attn_bwd_workspace_bytes": (I64, [P]),
        "ug_hier_local_attn_bwd": (I32, [P] + [P] * 17 + [P, I64, P]),
        "ug_hier_local_attn_bwd_vo_raster": (I32, [P] + [P] * 17 + [P, I64, P]),
        "ug_layer_bwd_workspace_bytes": (I64, [P]),
        "ug_layer_bwd": (I32, [P] + [P] * 17 + [P, I64, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _loaded[path] = L
    return L


def status_string(status: int) -> str:
    return lib().ug_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != UG_OK:
        raise UgError(status, what)


def make_geom(**kw) -> ug_geom:
    g = ug_geom()
    for name, _ in ug_geom._fields_:
        setattr(g, name, kw.get(name, 0))
    return g


def geom_validate(g: ug_geom) -> int:
    return lib().ug_geom_validate(ctypes.byref(g))


def build_index_maps(g: ug_geom):
    """(perm, nbr_off, nbr_idx) as int32 numpy arrays (host only)."""
    n = [ctypes.c_int64() for _ in range(3)]
    _check(lib().ug_index_map_sizes(ctypes.byref(g), *[ctypes.byref(x) for x in n]),
           "ug_index_map_sizes")
    arrs = [np.zeros(x.value, dtype=np.int32) for x in n]
    ptrs = [a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) for a in arrs]
    _check(lib().ug_build_index_maps(ctypes.byref(g), *ptrs), "ug_build_index_maps")
    return tuple(arrs)


def work_lists(g: ug_geom):
    """(qctas [n, 4], kvlist, kctas [m, 4], qlist) as numpy arrays (host only)."""
    n = [ctypes.c_int64() for _ in range(4)]
    _check(lib().ug_work_list_sizes(ctypes.byref(g), *[ctypes.byref(x) for x in n]),
           "ug_work_list_sizes")
    qc = np.zeros((n[0].value, 4), dtype=np.int32)
    kv = np.zeros(n[1].value, dtype=np.uint32)
    kc = np.zeros((n[2].value, 4), dtype=np.int32)
    ql = np.zeros(n[3].value, dtype=np.uint32)
    p32 = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    pu32 = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32))
    _check(lib().ug_build_work_lists(ctypes.byref(g), p32(qc), pu32(kv), p32(kc), pu32(ql)),
           "ug_build_work_lists")
    return qc, kv, kc, ql


def visible_pairs(g: ug_geom):
    """Per (batch, head): (hr_hr, hr_lr, lr_lr) visible query/key pairs."""
    n = [ctypes.c_int64() for _ in range(3)]
    _check(lib().ug_visible_pairs(ctypes.byref(g), *[ctypes.byref(x) for x in n]),
           "ug_visible_pairs")
    return tuple(x.value for x in n)


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    if not t.is_contiguous():
        raise ValueError("contiguous tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


class Plan:
    """Owns a ug_plan (device index lists and RoPE tables) for one geometry."""

    def __init__(self, **geom):
        self.geom_kw = dict(geom)
        self.g = make_geom(**geom)
        h = ctypes.c_void_p()
        self._L = lib()  # a plan is valid only in the library that created it
        _check(self._L.ug_plan_create(ctypes.byref(self.g), ctypes.byref(h)), "ug_plan_create")
        self.handle = h

    def close(self):
        if self.handle:
            _check(self._L.ug_plan_destroy(self.handle), "ug_plan_destroy")
            self.handle = None

    def __del__(self):
        try:
            if getattr(self, "handle", None):
                self._L.ug_plan_destroy(self.handle)
                self.handle = None
        except Exception:
            pass

    # -- host-side views ---------------------------------------------------
    def index_maps(self):
        n = [ctypes.c_int64() for _ in range(3)]
        _check(self._L.ug_index_map_sizes(ctypes.byref(self.g), *[ctypes.byref(x) for x in n]),
               "ug_index_map_sizes")
        arrs = [np.zeros(x.value, dtype=np.int32) for x in n]
        ptrs = [a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)) for a in arrs]
        _check(self._L.ug_get_index_maps(self.handle, *ptrs), "ug_get_index_maps")
        return tuple(arrs)

    def workspace_bytes(self) -> int:
        return int(self._L.ug_layer_workspace_bytes(self.handle))

    # -- the four steps --------------------------------------------------------
    def permute_window_first(self, src, dst, stream=None) -> int:
        return self._L.ug_permute_window_first(self.handle, _ptr(src), _ptr(dst), _stream(stream))

    def permute_rope_window_first(self, src, dst, stream=None) -> int:
        return self._L.ug_permute_rope_window_first(self.handle, _ptr(src), _ptr(dst),
                                                  _stream(stream))

    def unpermute(self, src, dst, stream=None) -> int:
        return self._L.ug_unpermute(self.handle, _ptr(src), _ptr(dst), _stream(stream))

    def rope_2d(self, x, y, token_set: int, stream=None) -> int:
        return self._L.ug_rope_2d(self.handle, _ptr(x), _ptr(y), int(token_set), _stream(stream))

    def hier_local_attn_fwd(self, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse=None,
                            stream=None) -> int:
        return self._L.ug_hier_local_attn_fwd(
            self.handle, _ptr(q_hr), _ptr(k_hr), _ptr(v_hr), _ptr(q_lr), _ptr(k_lr), _ptr(v_lr),
            _ptr(o_hr), _ptr(o_lr), _ptr(lse), _stream(stream))

    def hier_local_attn_fwd_vo_raster(self, q_hr, k_hr, v_hr_raster, q_lr, k_lr, v_lr,
                                      o_hr_raster, o_lr, lse=None, stream=None) -> int:
        return self._L.ug_hier_local_attn_fwd_vo_raster(
            self.handle, _ptr(q_hr), _ptr(k_hr), _ptr(v_hr_raster), _ptr(q_lr), _ptr(k_lr),
            _ptr(v_lr), _ptr(o_hr_raster), _ptr(o_lr), _ptr(lse), _stream(stream))

    def layer_fwd(self, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, workspace,
                  stream=None) -> int:
        return self._L.ug_layer_fwd(
            self.handle, _ptr(q_hr), _ptr(k_hr), _ptr(v_hr), _ptr(q_lr), _ptr(k_lr), _ptr(v_lr),
            _ptr(o_hr), _ptr(o_lr), _ptr(lse), _ptr(workspace),
            ctypes.c_int64(workspace.numel() * workspace.element_size()), _stream(stream))

    def layer_fwd_static_scratch(self, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse,
                                 stream=None) -> int:
        """The layer without a caller workspace: its intermediates live in the
        library's static device scratch (no device allocation on this call)."""
        return self._L.ug_layer_fwd_static_scratch(
            self.handle, _ptr(q_hr), _ptr(k_hr), _ptr(v_hr), _ptr(q_lr), _ptr(k_lr), _ptr(v_lr),
            _ptr(o_hr), _ptr(o_lr), _ptr(lse), _stream(stream))

    def set_wait_timeout(self, ns: int) -> int:
        return self._L.ug_plan_set_wait_timeout(self.handle, ctypes.c_int64(int(ns)))

    def check_error(self, stream=None) -> int:
        return self._L.ug_check_error(self.handle, _stream(stream))

    # -- backward ----------------------------------------------------------------
    def rope_2d_bwd(self, dy, dx, token_set: int, stream=None) -> int:
        return self._L.ug_rope_2d_bwd(self.handle, _ptr(dy), _ptr(dx), int(token_set),
                                    _stream(stream))

    def unpermute_rope_bwd(self, src_wf, dst_raster, stream=None) -> int:
        return self._L.ug_unpermute_rope_bwd(self.handle, _ptr(src_wf), _ptr(dst_raster),
                                           _stream(stream))

    def attn_bwd_workspace_bytes(self) -> int:
        return int(self._L.ug_attn_bwd_workspace_bytes(self.handle))

    def layer_bwd_workspace_bytes(self) -> int:
        return int(self._L.ug_layer_bwd_workspace_bytes(self.handle))

    def hier_local_attn_bwd(self, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr, do_lr,
                            lse, dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr, workspace,
                            stream=None) -> int:
        args = (q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr, do_lr, lse, dq_hr, dk_hr,
                dv_hr, dq_lr, dk_lr, dv_lr, workspace)
        return self._L.ug_hier_local_attn_bwd(
            self.handle, *[_ptr(a) for a in args],
            ctypes.c_int64(workspace.numel() * workspace.element_size()), _stream(stream))

    def hier_local_attn_bwd_vo_raster(self, q_hr, k_hr, v_hr_raster, q_lr, k_lr, v_lr,
                                      o_hr_raster, o_lr, do_hr_raster, do_lr, lse, dq_hr, dk_hr,
                                      dv_hr_raster, dq_lr, dk_lr, dv_lr, workspace,
                                      stream=None) -> int:
        args = (q_hr, k_hr, v_hr_raster, q_lr, k_lr, v_lr, o_hr_raster, o_lr, do_hr_raster,
                do_lr, lse, dq_hr, dk_hr, dv_hr_raster, dq_lr, dk_lr, dv_lr, workspace)
        return self._L.ug_hier_local_attn_bwd_vo_raster(
            self.handle, *[_ptr(a) for a in args],
            ctypes.c_int64(workspace.numel() * workspace.element_size()), _stream(stream))

    def layer_bwd(self, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, do_hr, do_lr,
                  dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr, workspace, stream=None) -> int:
        args = (q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, do_hr, do_lr, dq_hr, dk_hr,
                dv_hr, dq_lr, dk_lr, dv_lr, workspace)
        return self._L.ug_layer_bwd(
            self.handle, *[_ptr(a) for a in args],
            ctypes.c_int64(workspace.numel() * workspace.element_size()), _stream(stream))


# ---- convenience wrappers (allocate outputs with torch, raise on errors) -----

def permute_window_first(plan: Plan, x: torch.Tensor) -> torch.Tensor:
    out = torch.empty_like(x)
    _check(plan.permute_window_first(x, out), "ug_permute_window_first")
    return out


def permute_rope_window_first(plan: Plan, x: torch.Tensor) -> torch.Tensor:
    out = torch.empty_like(x)
    _check(plan.permute_rope_window_first(x, out), "ug_permute_rope_window_first")
    return out


def unpermute(plan: Plan, x: torch.Tensor) -> torch.Tensor:
    out = torch.empty_like(x)
    _check(plan.unpermute(x, out), "ug_unpermute")
    return out


def rope_2d(plan: Plan, x: torch.Tensor, token_set: int, inplace: bool = False) -> torch.Tensor:
    out = x if inplace else torch.empty_like(x)
    _check(plan.rope_2d(x, out, token_set), "ug_rope_2d")
    return out


def hier_local_attn_fwd(plan: Plan, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, want_lse=True):
    o_hr = torch.empty_like(q_hr)
    o_lr = torch.empty_like(q_lr) if q_lr is not None and q_lr.numel() else None
    lse = None
    if want_lse:
        B, N, H, _ = q_hr.shape
        L = q_lr.shape[1] if q_lr is not None else 0
        lse = torch.empty((B, H, N + L), dtype=torch.float32, device=q_hr.device)
    lr = (q_lr, k_lr, v_lr) if o_lr is not None else (None, None, None)
    _check(plan.hier_local_attn_fwd(q_hr, k_hr, v_hr, *lr, o_hr, o_lr, lse),
           "ug_hier_local_attn_fwd")
    return o_hr, o_lr, lse


def _like(x):
    return torch.empty_like(x) if x is not None and x.numel() else None


def hier_local_attn_bwd(plan: Plan, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr,
                        do_lr, lse):
    """Gradients of hier_local_attn_fwd; returns (dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr)."""
    outs = [_like(t) for t in (q_hr, k_hr, v_hr, q_lr, k_lr, v_lr)]
    ws = torch.empty(plan.attn_bwd_workspace_bytes(), dtype=torch.uint8, device=q_hr.device)
    _check(plan.hier_local_attn_bwd(q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, do_hr, do_lr,
                                    lse, *outs, ws), "ug_hier_local_attn_bwd")
    return tuple(outs)


def layer_backward(plan: Plan, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, do_hr, do_lr,
                   workspace=None):
    """Gradients of layer_forward w.r.t. its raster inputs; returns
    (dq_hr, dk_hr, dv_hr, dq_lr, dk_lr, dv_lr)."""
    if workspace is None:
        workspace = torch.empty(plan.layer_bwd_workspace_bytes(), dtype=torch.uint8,
                                device=q_hr.device)
    outs = [_like(t) for t in (q_hr, k_hr, v_hr, q_lr, k_lr, v_lr)]
    _check(plan.layer_bwd(q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, o_hr, o_lr, lse, do_hr, do_lr,
                          *outs, workspace), "ug_layer_bwd")
    return tuple(outs)


def rope_2d_bwd(plan: Plan, dy: torch.Tensor, token_set: int) -> torch.Tensor:
    out = torch.empty_like(dy)
    _check(plan.rope_2d_bwd(dy, out, token_set), "ug_rope_2d_bwd")
    return out


def unpermute_rope_bwd(plan: Plan, x: torch.Tensor) -> torch.Tensor:
    out = torch.empty_like(x)
    _check(plan.unpermute_rope_bwd(x, out), "ug_unpermute_rope_bwd")
    return out


def warm_start_raw(x_lr: torch.Tensor, noise: torch.Tensor, out: torch.Tensor, scale: int,
                   sharpen: float, t: float, stream=None) -> int:
    """ug_warm_start on fp32 [B, C, h, w] / [B, C, h*s, w*s] device tensors;
    returns the status."""
    B, C, h, w = x_lr.shape
    prm = ug_warm_start_params(B, C, h, w, int(scale), float(sharpen), float(t))
    return lib().ug_warm_start(ctypes.byref(prm), _ptr(x_lr), _ptr(noise), _ptr(out),
                               _stream(stream))


def warm_start_stencil_weights(sharpen: float, t: float):
    """ug_warm_start_stencil_weights (host only): the factor-4 warm start's
    weights as a [4, 4, 3, 3] numpy array ([py, px, r, c])."""
    w = np.zeros(144, dtype=np.float32)
    _check(lib().ug_warm_start_stencil_weights(
        float(sharpen), float(t), w.ctypes.data_as(ctypes.POINTER(ctypes.c_float))),
        "ug_warm_start_stencil_weights")
    return w.reshape(4, 4, 3, 3)


def warm_start(x_lr: torch.Tensor, noise: torch.Tensor, scale: int, sharpen: float, t: float,
               out: torch.Tensor = None) -> torch.Tensor:
    """(1 - t) * sharpen(upsample(x_lr)) + t * noise, into a new tensor (or out)."""
    out = torch.empty_like(noise) if out is None else out
    _check(warm_start_raw(x_lr, noise, out, scale, sharpen, t), "ug_warm_start")
    return out


def layer_forward(plan: Plan, q_hr, k_hr, v_hr, q_lr, k_lr, v_lr, workspace=None, want_lse=True):
    """Whole layer on raster-order device tensors; returns (o_hr raster, o_lr, lse)."""
    if workspace is None:
        workspace = torch.empty(plan.workspace_bytes(), dtype=torch.uint8, device=q_hr.device)
    o_hr = torch.empty_like(q_hr)
    has_lr = q_lr is not None and q_lr.numel() > 0
    o_lr = torch.empty_like(q_lr) if has_lr else None
    lse = None
    if want_lse:
        B, N, H, _ = q_hr.shape
        L = q_lr.shape[1] if has_lr else 0
        lse = torch.empty((B, H, N + L), dtype=torch.float32, device=q_hr.device)
    lr = (q_lr, k_lr, v_lr) if has_lr else (None, None, None)
    _check(plan.layer_fwd(q_hr, k_hr, v_hr, *lr, o_hr, o_lr, lse, workspace), "ug_layer_fwd")
    return o_hr, o_lr, lse
