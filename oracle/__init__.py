"""CPU oracle for the routed int4 MoE layer -- TEST INFRASTRUCTURE ONLY.

Python access to ``moe_oracle.c`` (plain scalar C, double accumulation).  Only the test
suite, the package smoke check and the benchmark's CPU-baseline leg may import this
package.  The CUDA library never imports, links or calls it, and the two share no code.

Every function takes and returns numpy arrays.  Building the shared library needs only
``gcc`` and libm.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libmoe_oracle.so")
_lock = threading.Lock()
_lib = None

# gcc flags: no fast-math and no floating-point contraction, so every sum is the plain
# left-to-right double sum the C source spells out.
CFLAGS = ["-O2", "-std=c11", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into oracle/_build/libmoe_oracle.so (if stale)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i32, i64, dbl = ctypes.c_int, ctypes.c_int64, ctypes.c_double
            L.orc_nibble.argtypes = [P, i64]
            L.orc_nibble.restype = i32
            L.orc_half.argtypes = [ctypes.c_uint16]
            L.orc_half.restype = dbl
            L.orc_bf16_round.argtypes = [ctypes.c_float]
            L.orc_bf16_round.restype = ctypes.c_float
            L.orc_blob_bytes.argtypes = [i32, i32]
            L.orc_blob_bytes.restype = i64
            L.orc_blob_weight.argtypes = [i32, i32, P, i32, i64, i64, i32]
            L.orc_blob_weight.restype = dbl
            L.orc_expert.argtypes = [i32, i32, P, P, i32, P, P]
            L.orc_expert.restype = i32
            L.orc_route.argtypes = [i32, i32, i32, i32, P, P, P, P, P, P]
            L.orc_route.restype = i32
            L.orc_union.argtypes = [i32, i32, i32, P, P, P, P, P]
            L.orc_union.restype = i32
            L.orc_forward.argtypes = [i32, i32, i32, i32, i32, i32, P, P, i64, P, P, P, i32, P]
            L.orc_forward.restype = i32
            L.orc_rmsnorm.argtypes = [i32, i32, P, P, dbl, P]
            L.orc_rmsnorm.restype = i32
            L.orc_crumb.argtypes = [P, i64]
            L.orc_crumb.restype = i32
            L.orc_int8.argtypes = [P, i64]
            L.orc_int8.restype = i32
            L.orc_blob_bytes_fmt.argtypes = [i32, i32, i32]
            L.orc_blob_bytes_fmt.restype = i64
            L.orc_blob_weight_fmt.argtypes = [i32, i32, i32, P, i32, i64, i64]
            L.orc_blob_weight_fmt.restype = dbl
            L.orc_expert_fmt.argtypes = [i32, i32, i32, P, P, P]
            L.orc_expert_fmt.restype = i32
            L.orc_forward_fmt.argtypes = [i32, i32, i32, i32, i32, i32, i32, P, P, i64, P, P, P, P]
            L.orc_forward_fmt.restype = i32
            _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: oracle status {rc}")


# ------------------------------------------------------------------------------------
# Thin wrappers
# ------------------------------------------------------------------------------------

def nibble(row: np.ndarray, c: int) -> int:
    row = _c(row, np.uint8)
    return lib().orc_nibble(_ptr(row), c)


def half(bits: int) -> float:
    return lib().orc_half(bits)


def bf16_round(v: float) -> float:
    return lib().orc_bf16_round(v)


def blob_bytes(H: int, I: int) -> int:
    return lib().orc_blob_bytes(H, I)


def blob_weight(H, I, blob, which, r, c, bf16=False) -> float:
    blob = _c(blob, np.uint8)
    return lib().orc_blob_weight(H, I, _ptr(blob), which, r, c, int(bf16))


def expert(H, I, blob, x, bf16=False):
    """One expert on one token -> (out [H] float64, h [I] float64).

    bf16: False/0 fp32 contract; True/1 bf16 weights and bf16 h; 2 bf16 weights, exact h.
    """
    blob = _c(blob, np.uint8)
    x = _c(x, np.float32)
    out = np.zeros(H, np.float64)
    h = np.zeros(I, np.float64)
    _check(lib().orc_expert(H, I, _ptr(blob), _ptr(x), int(bf16), _ptr(out), _ptr(h)),
           "expert")
    return out, h


def route(x, w_router, bias, k):
    """-> (idx [T][k] int32, w [T][k] float32, logits [T][E] float32)."""
    x = _c(x, np.float32)
    w_router = _c(w_router, np.float32)
    T, H = x.shape
    E = w_router.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    logits = np.zeros((T, E), np.float32)
    _check(lib().orc_route(H, E, k, T, _ptr(x), _ptr(w_router), _ptr(b), _ptr(idx), _ptr(w),
                           _ptr(logits)), "route")
    return idx, w, logits


def union(idx, n_experts):
    """-> (union_ids [E], n_union, offsets [E+1], assign [T*k]) as int32."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    E = n_experts
    uid = np.zeros(E, np.int32)
    nu = np.zeros(1, np.int32)
    off = np.zeros(E + 1, np.int32)
    asg = np.zeros(max(T * k, 1), np.int32)[:T * k]
    _check(lib().orc_union(E, k, T, _ptr(idx), _ptr(uid), _ptr(nu), _ptr(off), _ptr(asg)),
           "union")
    return uid, int(nu[0]), off, asg


def forward(H, I, E, k, n_shared, x, experts, stride, shared, idx, w, bf16=False):
    """y [T][H] float32.  experts: uint8 array holding E blobs `stride` bytes apart."""
    x = _c(x, np.float32)
    T = x.shape[0]
    experts = _c(experts, np.uint8)
    sh = None if shared is None else _c(shared, np.uint8)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    y = np.zeros((T, H), np.float32)
    _check(lib().orc_forward(H, I, E, k, n_shared, T, _ptr(x), _ptr(experts), stride, _ptr(sh),
                             _ptr(idx), _ptr(w), int(bf16), _ptr(y)), "forward")
    return y


# weight containers (orc_forward_fmt): gs64 int4, gs64 int8, per-row int4, gs64 int2
FMT_INT4_G64, FMT_INT8_G64, FMT_INT4_ROW, FMT_INT2_G64 = 0, 1, 2, 3


def crumb(row: np.ndarray, c: int) -> int:
    row = _c(row, np.uint8)
    return lib().orc_crumb(_ptr(row), c)


def int8_value(row: np.ndarray, c: int) -> int:
    row = _c(row, np.uint8)
    return lib().orc_int8(_ptr(row), c)


def blob_bytes_fmt(H: int, I: int, fmt: int) -> int:
    return lib().orc_blob_bytes_fmt(H, I, fmt)


def blob_weight_fmt(H, I, fmt, blob, which, r, c) -> float:
    blob = _c(blob, np.uint8)
    return lib().orc_blob_weight_fmt(H, I, fmt, _ptr(blob), which, r, c)


def forward_fmt(H, I, E, k, n_shared, fmt, x, experts, stride, shared, idx, w):
    """y [T][H] float32 for blobs in container fmt (fp32 contract)."""
    x = _c(x, np.float32)
    T = x.shape[0]
    experts = _c(experts, np.uint8)
    sh = None if shared is None else _c(shared, np.uint8)
    idx = _c(idx, np.int32)
    w = _c(w, np.float32)
    y = np.zeros((T, H), np.float32)
    _check(lib().orc_forward_fmt(H, I, E, k, n_shared, T, fmt, _ptr(x), _ptr(experts), stride, _ptr(sh),
                                 _ptr(idx), _ptr(w), _ptr(y)), "forward_fmt")
    return y


def forward_sparse_fmt(H, I, k, n_shared, fmt, x, blobs: dict, shared, idx, w):
    """forward_fmt for tokens whose experts are given as a dict {expert_id: blob}."""
    ids = sorted(blobs)
    remap = {e: j for j, e in enumerate(ids)}
    nb = len(blobs[ids[0]])
    packed = np.zeros((len(ids), nb), np.uint8)
    for j, e in enumerate(ids):
        packed[j] = np.asarray(blobs[e], np.uint8)
    idx2 = np.vectorize(lambda e: remap[int(e)])(np.asarray(idx)).astype(np.int32)
    return forward_fmt(H, I, len(ids), k, n_shared, fmt, x, packed, nb, shared, idx2, w)


def forward_sparse(H, I, k, n_shared, x, blobs: dict, shared, idx, w, bf16=False):
    """Forward for tokens whose experts are given as a dict {expert_id: blob}.

    Used at full size, where only the selected experts are regenerated on the host.
    The dict's blobs are packed into a compact array and idx is renumbered into it;
    the arithmetic is orc_forward's.
    """
    ids = sorted(blobs)
    remap = {e: j for j, e in enumerate(ids)}
    nb = len(blobs[ids[0]])
    packed = np.zeros((len(ids), nb), np.uint8)
    for j, e in enumerate(ids):
        packed[j] = np.asarray(blobs[e], np.uint8)
    idx2 = np.vectorize(lambda e: remap[int(e)])(np.asarray(idx)).astype(np.int32)
    return forward(H, I, len(ids), k, n_shared, x, packed, nb, shared, idx2, w, bf16)


def rmsnorm(x, gamma, eps=1e-5):
    x = _c(x, np.float32)
    T, H = x.shape
    g = _c(gamma, np.float32)
    out = np.zeros_like(x)
    _check(lib().orc_rmsnorm(H, T, _ptr(x), _ptr(g), eps, _ptr(out)), "rmsnorm")
    return out


# ------------------------------------------------------------------------------------
# Composition: one layer, and a residual layer stack
# ------------------------------------------------------------------------------------

def layer(H, I, E, k, n_shared, x, w_router, bias, experts, stride, shared, bf16=False):
    """route -> union -> forward for one batch.  Returns a dict of every result."""
    idx, w, logits = route(x, w_router, bias, k)
    uid, nu, off, asg = union(idx, E)
    y = forward(H, I, E, k, n_shared, x, experts, stride, shared, idx, w, bf16)
    return dict(idx=idx, w=w, logits=logits, union_ids=uid, n_union=nu, offsets=off,
                assign=asg, y=y)


def stack_layer(x, gamma, eps, w_router, bias, k, H, I, n_shared, get_blob, shared,
                bf16=False):
    """One residual layer: n = RMSNorm(x); x_out = x + MoE(n), float32 add.

    get_blob(e) returns expert e's blob (so only selected experts are materialised).
    Returns (x_out, n, idx, w, logits, y).
    """
    n = rmsnorm(x, gamma, eps)
    idx, w, logits = route(n, w_router, bias, k)
    blobs = {int(e): get_blob(int(e)) for e in np.unique(idx)}
    y = forward_sparse(H, I, k, n_shared, n, blobs, shared, idx, w, bf16)
    x_out = (x.astype(np.float32) + y.astype(np.float32)).astype(np.float32)
    return x_out, n, idx, w, logits, y
