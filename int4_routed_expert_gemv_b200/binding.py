"""Thin Python binding of libcolimoe.so (ctypes).

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
Functions keep the C names and take torch tensors (device memory) in place of pointers;
each returns the library's status code.  `check()` turns a status into an exception.
The shared library must exist (built by ``int4_routed_expert_gemv_b200.build``); there is
no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libcolimoe.so")

COLI_OK, COLI_EINVAL, COLI_ENOMEM, COLI_ECUDA, COLI_ETIMEOUT, COLI_EUNSUPPORTED, COLI_EDEVICE = range(7)
COLI_F32, COLI_BF16 = 0, 1
DEV_NONFINITE, DEV_BAD_INDEX, DEV_TIMEOUT, DEV_BAD_SHAPE = 1, 2, 4, 8

EXPORTS = [
    "coli_moe_blob_bytes", "coli_moe_workspace_bytes", "coli_moe_workspace_init",
    "coli_moe_read_status", "coli_moe_route", "coli_moe_route_union", "coli_moe_union", "coli_moe_forward",
    "coli_moe_gate_up", "coli_moe_down", "coli_moe_layer", "coli_moe_stack", "coli_rmsnorm",
    "coli_moe_forward_noalloc", "coli_moe_noalloc_read_status", "coli_debug_wait_timeout",
    "coli_debug_phase_stamps",
    "coli_moe_blob_bytes_fmt", "coli_moe_forward_fmt", "coli_moe_union_restrict",
    "coli_status_string",
]


class Dims(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32),
                ("n_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("n_shared", ctypes.c_int32)]


class Weights(ctypes.Structure):
    _fields_ = [("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("experts", ctypes.c_void_p), ("shared", ctypes.c_void_p),
                ("expert_stride", ctypes.c_size_t)]


class ColiError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


_lock = threading.Lock()
_lib = None


def lib():
    """Load libcolimoe.so; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m int4_routed_expert_gemv_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
            D, W = ctypes.POINTER(Dims), ctypes.POINTER(Weights)
            sig = {
                "coli_moe_blob_bytes": (sz, [i32, i32]),
                "coli_moe_workspace_bytes": (sz, [D, i32]),
                "coli_moe_workspace_init": (i32, [P, sz, P]),
                "coli_moe_read_status": (i32, [P, ctypes.POINTER(ctypes.c_uint32), P]),
                "coli_moe_route": (i32, [D, P, P, P, i32, i32, P, P, P, P, sz, P]),
                "coli_moe_union": (i32, [D, P, i32, P, P, P, P, P, sz, P]),
                "coli_moe_route_union": (i32, [D, P, P, P, i32, i32, P, P, P, P, P, P, P, P, sz, P]),
                "coli_moe_forward": (i32, [D, W, P, i32, i32, P, P, P, P, P, P, P, P, P, sz, P]),
                "coli_moe_gate_up": (i32, [D, W, P, i32, P, P, P, P, P, sz, P]),
                "coli_moe_down": (i32, [D, W, i32, P, P, P, P, P, P, P, P, sz, P]),
                "coli_moe_layer": (i32, [D, W, P, i32, i32, P, P, P, P, P, P, P, P, P, P, sz, P]),
                "coli_moe_stack": (i32, [D, W, P, i32, ctypes.c_double, P, i32, P, P, P, sz, P]),
                "coli_rmsnorm": (i32, [i32, i32, P, P, ctypes.c_double, P, P]),
                "coli_moe_forward_noalloc": (i32, [D, W, P, i32, P, P, P, P, P, P, P, P]),
                "coli_moe_noalloc_read_status": (i32, [ctypes.POINTER(ctypes.c_uint32), P]),
                "coli_debug_wait_timeout": (i32, [P, sz, ctypes.c_uint64, P, P]),
                "coli_debug_phase_stamps": (i32, [P, i32, P, P]),
                "coli_moe_blob_bytes_fmt": (sz, [i32, i32, i32]),
                "coli_moe_union_restrict": (i32, [D, i32, i32, i32, P, P, P, P, P, P, P, P, P]),
                "coli_moe_forward_fmt": (i32, [D, i32, W, P, i32, P, P, P, P, P, P, P, P, sz, P]),
                "coli_status_string": (ctypes.c_char_p, [i32]),
            }
            for name, (res, args) in sig.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().coli_status_string(int(s)).decode()


def check(status: int, what: str = "colimoe") -> None:
    if status != COLI_OK:
        raise ColiError(status, what)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dt(x: torch.Tensor) -> int:
    if x.dtype == torch.float32:
        return COLI_F32
    if x.dtype == torch.bfloat16:
        return COLI_BF16
    raise TypeError(f"unsupported activation dtype {x.dtype}")


def make_dims(hidden, inter, n_experts, top_k, n_shared=1) -> Dims:
    return Dims(hidden, inter, n_experts, top_k, n_shared)


def make_weights(w_router, router_bias, experts, shared, expert_stride) -> Weights:
    return Weights(_p(w_router), _p(router_bias), _p(experts), _p(shared), int(expert_stride))


def coli_moe_blob_bytes(hidden: int, inter: int) -> int:
    return lib().coli_moe_blob_bytes(hidden, inter)


def coli_moe_workspace_bytes(dims: Dims, T_max: int) -> int:
    return lib().coli_moe_workspace_bytes(ctypes.byref(dims), T_max)


def coli_moe_workspace_init(ws: torch.Tensor, stream=None) -> int:
    return lib().coli_moe_workspace_init(_p(ws), ws.numel() * ws.element_size(), _s(stream))


FMT_INT4_G64, FMT_INT8_G64, FMT_INT4_ROW, FMT_INT2_G64 = 0, 1, 2, 3


def coli_moe_blob_bytes_fmt(hidden: int, inter: int, fmt: int) -> int:
    return int(lib().coli_moe_blob_bytes_fmt(hidden, inter, fmt))


def coli_moe_forward_fmt(dims, fmt, weights, x, T, w, union_ids, n_union, offsets, assign, residual, y, ws,
                         stream=None) -> int:
    return lib().coli_moe_forward_fmt(ctypes.byref(dims), int(fmt), ctypes.byref(weights), _p(x), T, _p(w),
                                      _p(union_ids), _p(n_union), _p(offsets), _p(assign), _p(residual), _p(y),
                                      _p(ws), ws.numel(), _s(stream))


def coli_moe_union_restrict(dims, T, e0, e1, union_ids, n_union, offsets, assign, union_ids_l, n_union_l,
                            offsets_l, assign_l, stream=None) -> int:
    return lib().coli_moe_union_restrict(ctypes.byref(dims), T, e0, e1, _p(union_ids), _p(n_union), _p(offsets),
                                         _p(assign), _p(union_ids_l), _p(n_union_l), _p(offsets_l), _p(assign_l),
                                         _s(stream))


def coli_moe_noalloc_read_status(stream=None):
    v = ctypes.c_uint32(0)
    st = lib().coli_moe_noalloc_read_status(ctypes.byref(v), _s(stream))
    return st, int(v.value)


def coli_debug_wait_timeout(ws: torch.Tensor, budget_cycles: int, returned: torch.Tensor, stream=None) -> int:
    return lib().coli_debug_wait_timeout(_p(ws), ws.numel(), int(budget_cycles), _p(returned), _s(stream))


def coli_debug_phase_stamps(max_ctas: int = 256):
    """(status, stamps [n_ctas][n_stamps] as a numpy uint64 array) of the last fused launch."""
    import numpy as np
    buf = np.zeros((max_ctas, 16), np.uint64)
    n_ctas, n_st = ctypes.c_int32(0), ctypes.c_int32(0)
    st = lib().coli_debug_phase_stamps(buf.ctypes.data, max_ctas, ctypes.byref(n_ctas), ctypes.byref(n_st))
    return st, buf[:n_ctas.value, :n_st.value]


def coli_moe_read_status(ws: torch.Tensor, stream=None):
    v = ctypes.c_uint32(0)
    st = lib().coli_moe_read_status(_p(ws), ctypes.byref(v), _s(stream))
    return st, int(v.value)


def coli_moe_route(dims, w_router, bias, x, T, idx, w, logits, ws, stream=None) -> int:
    return lib().coli_moe_route(ctypes.byref(dims), _p(w_router), _p(bias), _p(x), _dt(x), T,
                                _p(idx), _p(w), _p(logits), _p(ws), ws.numel(), _s(stream))


def coli_moe_route_union(dims, w_router, bias, x, T, idx, w, logits, union_ids, n_union,
                         offsets, assign, ws, stream=None) -> int:
    return lib().coli_moe_route_union(ctypes.byref(dims), _p(w_router), _p(bias), _p(x), _dt(x),
                                      T, _p(idx), _p(w), _p(logits), _p(union_ids), _p(n_union),
                                      _p(offsets), _p(assign), _p(ws), ws.numel(), _s(stream))


def coli_moe_union(dims, idx, T, union_ids, n_union, offsets, assign, ws, stream=None) -> int:
    return lib().coli_moe_union(ctypes.byref(dims), _p(idx), T, _p(union_ids), _p(n_union),
                                _p(offsets), _p(assign), _p(ws), ws.numel(), _s(stream))


def coli_moe_forward(dims, weights, x, T, idx, w, union_ids, n_union, offsets, assign,
                     residual, y, ws, stream=None) -> int:
    return lib().coli_moe_forward(ctypes.byref(dims), ctypes.byref(weights), _p(x), _dt(x), T,
                                  _p(idx), _p(w), _p(union_ids), _p(n_union), _p(offsets),
                                  _p(assign), _p(residual), _p(y), _p(ws), ws.numel(), _s(stream))


def coli_moe_gate_up(dims, weights, x, T, union_ids, n_union, offsets, assign, ws,
                     stream=None) -> int:
    return lib().coli_moe_gate_up(ctypes.byref(dims), ctypes.byref(weights), _p(x), T,
                                  _p(union_ids), _p(n_union), _p(offsets), _p(assign), _p(ws),
                                  ws.numel(), _s(stream))


def coli_moe_down(dims, weights, T, w, union_ids, n_union, offsets, assign, residual, y, ws,
                  stream=None) -> int:
    return lib().coli_moe_down(ctypes.byref(dims), ctypes.byref(weights), T, _p(w),
                               _p(union_ids), _p(n_union), _p(offsets), _p(assign),
                               _p(residual), _p(y), _p(ws), ws.numel(), _s(stream))


def coli_moe_layer(dims, weights, x, T, idx, w, logits, union_ids, n_union, offsets, assign,
                   residual, y, ws, stream=None) -> int:
    return lib().coli_moe_layer(ctypes.byref(dims), ctypes.byref(weights), _p(x), _dt(x), T,
                                _p(idx), _p(w), _p(logits), _p(union_ids), _p(n_union),
                                _p(offsets), _p(assign), _p(residual), _p(y), _p(ws),
                                ws.numel(), _s(stream))


def coli_moe_forward_noalloc(dims, weights, x, T, w, union_ids, n_union, offsets, assign,
                             residual, y, stream=None) -> int:
    """Forward without a workspace: scratch lives in a fixed 4 MiB array of the library's
    device memory, for callers that cannot allocate (see include/colimoe.h)."""
    return lib().coli_moe_forward_noalloc(ctypes.byref(dims), ctypes.byref(weights), _p(x), T,
                                          _p(w), _p(union_ids), _p(n_union), _p(offsets),
                                          _p(assign), _p(residual), _p(y), _s(stream))


def coli_moe_stack(dims, layers, gammas, eps, x, T, idx, y, ws, stream=None) -> int:
    """layers: list of Weights (one per layer); gammas: list of [H] device tensors or None
    (all-ones RMSNorm weights); idx: [L][T][k] int32 device tensor or None."""
    n = len(layers)
    arr = (Weights * max(n, 1))(*layers)
    if gammas is None:
        garr = None
    else:
        garr = (ctypes.c_void_p * max(n, 1))(*[None if g is None else g.data_ptr() for g in gammas])
    return lib().coli_moe_stack(ctypes.byref(dims), arr, garr, n, float(eps), _p(x), T, _p(idx),
                                _p(y), _p(ws), ws.numel(), _s(stream))


def coli_rmsnorm(hidden, T, x, gamma, eps, out, stream=None) -> int:
    return lib().coli_rmsnorm(hidden, T, _p(x), _p(gamma), float(eps), _p(out), _s(stream))


# ------------------------------------------------------------------------------------
# Buffers for one layer call (device allocations made by torch, owned by the caller)
# ------------------------------------------------------------------------------------

class LayerBuffers:
    """Device buffers for route/union/forward outputs of batches up to T_max tokens."""

    def __init__(self, dims: Dims, T_max: int, device="cuda"):
        E, k, H = dims.n_experts, dims.top_k, dims.hidden
        self.dims = dims
        self.T_max = T_max
        i32 = dict(dtype=torch.int32, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.idx = torch.zeros(max(T_max, 1), k, **i32)
        self.w = torch.zeros(max(T_max, 1), k, **f32)
        self.logits = torch.zeros(max(T_max, 1), E, **f32)
        self.union_ids = torch.zeros(E, **i32)
        self.n_union = torch.zeros(4, **i32)
        self.offsets = torch.zeros(E + 1, **i32)
        self.assign = torch.zeros(max(T_max * k, 1), **i32)
        self.y = torch.zeros(max(T_max, 1), H, **f32)
        nbytes = coli_moe_workspace_bytes(dims, T_max)
        if nbytes == 0:
            raise ValueError("invalid layer dimensions")
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        check(coli_moe_workspace_init(self.ws), "workspace_init")
