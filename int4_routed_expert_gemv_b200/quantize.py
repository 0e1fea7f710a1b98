"""Host-side quantisation of fp32 expert weights into the library's blob containers.

Symmetric absmax scaling, round to nearest (ties to even), clipped to the container's code
range:
  gs64 int4: one fp16 scale per 64 input columns, codes [-8, 7],     scale = absmax / 7;
  gs64 int8: one fp16 scale per 64 input columns, codes [-128, 127], scale = absmax / 127;
  per-row int4: one fp16 scale per row,           codes [-8, 7],     scale = absmax / 7;
  gs64 int2: one fp16 scale per 64 input columns, codes [-2, 1],     scale = absmax / 2.
The scale is rounded to fp16 first and the codes are taken against the rounded scale.  Blob
order: Gq | Uq | Dq | Gs | Us | Ds, payload packed with the lowest-index column in the
lowest bits (the layout of coli_moe_blob_bytes_fmt).  This is a weight preparation tool;
the forward itself runs on the GPU only.
"""
import numpy as np

FMT_INT4_G64, FMT_INT8_G64, FMT_INT4_ROW, FMT_INT2_G64 = 0, 1, 2, 3
BITS = {FMT_INT4_G64: 4, FMT_INT8_G64: 8, FMT_INT4_ROW: 4, FMT_INT2_G64: 2}
QRANGE = {FMT_INT4_G64: (-8, 7), FMT_INT8_G64: (-128, 127), FMT_INT4_ROW: (-8, 7), FMT_INT2_G64: (-2, 1)}
QDIV = {FMT_INT4_G64: 7.0, FMT_INT8_G64: 127.0, FMT_INT4_ROW: 7.0, FMT_INT2_G64: 2.0}


def quantize_matrix(W: np.ndarray, fmt: int):
    """W [rows][in] float -> (codes [rows][in] int8, scales [rows][in/64] or [rows][1] fp16)."""
    W = np.asarray(W, np.float32)
    rows, cols = W.shape
    assert cols % 64 == 0
    g = 1 if fmt == FMT_INT4_ROW else cols // 64
    Wg = W.reshape(rows, g, cols // g)
    amax = np.abs(Wg).max(axis=2)
    s16 = (amax / QDIV[fmt]).astype(np.float16)
    s = s16.astype(np.float32)
    safe = np.where(s > 0, s, 1.0)
    lo, hi = QRANGE[fmt]
    q = np.clip(np.rint(Wg / safe[:, :, None]), lo, hi)
    q = np.where(s[:, :, None] > 0, q, 0).astype(np.int8).reshape(rows, cols)
    return q, s16


def dequantize_matrix(q: np.ndarray, s16: np.ndarray) -> np.ndarray:
    rows, cols = q.shape
    g = s16.shape[1]
    return (q.reshape(rows, g, cols // g).astype(np.float32) * s16.astype(np.float32)[:, :, None]).reshape(rows, cols)


def pack_codes(q: np.ndarray, bits: int) -> np.ndarray:
    rows, cols = q.shape
    per = 8 // bits
    mask = (1 << bits) - 1
    u = (q.astype(np.int64) & mask).reshape(rows, cols // per, per)
    out = np.zeros((rows, cols // per), np.int64)
    for j in range(per):
        out |= u[:, :, j] << (bits * j)
    return out.astype(np.uint8).reshape(-1)


def expert_blob(G: np.ndarray, U: np.ndarray, D: np.ndarray, fmt: int):
    """G, U [I][H] and D [H][I] float -> (blob uint8, dequantised (G, U, D))."""
    parts, scs, deq = [], [], []
    for M in (G, U, D):
        q, s = quantize_matrix(M, fmt)
        parts.append(pack_codes(q, BITS[fmt]))
        scs.append(s.view(np.uint8).reshape(-1))
        deq.append(dequantize_matrix(q, s))
    return np.concatenate(parts + scs), tuple(deq)
