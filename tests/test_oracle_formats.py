"""Pins of the oracle's other weight containers (orc_*_fmt), CPU only.

Fixed against things other than the new code itself:
  * codecs: every int8 value and every 4-tuple of int2 values survives packing with plain
    two's-complement masks followed by the oracle's decoding;
  * byte counts: the closed forms of the blob sizes;
  * layouts and scale axes, through exact identities with the gs64 int4 oracle (pinned in
    test_oracle.py): an int8 or int2 blob holding values that int4 can hold gives exactly
    the int4 blob's y; a per-row blob gives exactly the y of a gs64 blob whose groups all
    carry the row's scale; container 0 through orc_forward_fmt is orc_forward.
A slip in a codec, an offset, a row stride or a scale index breaks one of these.
"""
import numpy as np
import pytest

import oracle
from oracle import FMT_INT2_G64, FMT_INT4_G64, FMT_INT4_ROW, FMT_INT8_G64

H, I, E, K = 128, 64, 4, 2
BITS = {FMT_INT4_G64: 4, FMT_INT8_G64: 8, FMT_INT4_ROW: 4, FMT_INT2_G64: 2}


def pack(q: np.ndarray, bits: int) -> np.ndarray:
    """Rows of signed values -> packed bytes, lowest column in the lowest bits."""
    rows, cols = q.shape
    per = 8 // bits
    mask = (1 << bits) - 1
    u = (q.astype(np.int64) & mask).reshape(rows, cols // per, per)
    out = np.zeros((rows, cols // per), np.int64)
    for j in range(per):
        out |= u[:, :, j] << (bits * j)
    return out.astype(np.uint8).reshape(-1)


def blob(fmt, qg, qu, qd, sg, su, sd) -> np.ndarray:
    b = BITS[fmt]
    parts = [pack(qg, b), pack(qu, b), pack(qd, b),
             sg.astype(np.float16).view(np.uint8).reshape(-1),
             su.astype(np.float16).view(np.uint8).reshape(-1),
             sd.astype(np.float16).view(np.uint8).reshape(-1)]
    out = np.concatenate(parts)
    assert out.size == oracle.blob_bytes_fmt(H, I, fmt)
    return out


def rand_expert(rng, lo, hi, fmt):
    qg = rng.integers(lo, hi + 1, (I, H))
    qu = rng.integers(lo, hi + 1, (I, H))
    qd = rng.integers(lo, hi + 1, (H, I))
    ng, nd = (1, 1) if fmt == FMT_INT4_ROW else (H // 64, I // 64)
    sg = rng.uniform(0.005, 0.02, (I, ng))
    su = rng.uniform(0.005, 0.02, (I, ng))
    sd = rng.uniform(0.005, 0.02, (H, nd))
    return qg, qu, qd, sg, su, sd


def layer(blobs, shared, fmt, x, idx, w):
    stride = blobs[0].size
    return oracle.forward_fmt(H, I, E, K, 1, fmt, x, np.concatenate(blobs), stride, shared, idx, w)


def inputs(rng, T=3):
    x = rng.standard_normal((T, H)).astype(np.float32)
    idx = np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)
    w = rng.dirichlet(np.ones(K), T).astype(np.float32)
    return x, idx, w


def test_int8_codec_every_value():
    vals = np.arange(-128, 128)
    row = (vals & 0xFF).astype(np.uint8)
    assert [oracle.int8_value(row, c) for c in range(256)] == vals.tolist()


def test_int2_codec_every_tuple():
    tuples = np.array([[a, b, c, d] for a in range(-2, 2) for b in range(-2, 2)
                       for c in range(-2, 2) for d in range(-2, 2)])
    row = pack(tuples, 2)
    assert row.size == 256 and len(set(row.tolist())) == 256
    got = np.array([oracle.crumb(row, c) for c in range(4 * 256)]).reshape(256, 4)
    assert np.array_equal(got, tuples)


@pytest.mark.parametrize("h,i", [(1024, 512), (6144, 2048)])
def test_blob_bytes_closed_forms(h, i):
    assert oracle.blob_bytes_fmt(h, i, FMT_INT4_G64) == oracle.blob_bytes(h, i)
    assert oracle.blob_bytes_fmt(h, i, FMT_INT8_G64) == 3 * h * i + 6 * h * i // 64
    assert oracle.blob_bytes_fmt(h, i, FMT_INT4_ROW) == 3 * h * i // 2 + 2 * (2 * i + h)
    assert oracle.blob_bytes_fmt(h, i, FMT_INT2_G64) == 3 * h * i // 4 + 6 * h * i // 64
    assert oracle.blob_bytes_fmt(h, i, 4) == -1


def test_container0_is_the_gs64_oracle():
    rng = np.random.default_rng(1)
    ex = [blob(FMT_INT4_G64, *rand_expert(rng, -8, 7, FMT_INT4_G64)) for _ in range(E)]
    sh = blob(FMT_INT4_G64, *rand_expert(rng, -8, 7, FMT_INT4_G64))
    x, idx, w = inputs(rng)
    y_fmt = layer(ex, sh, FMT_INT4_G64, x, idx, w)
    y_ref = oracle.forward(H, I, E, K, 1, x, np.concatenate(ex), ex[0].size, sh, idx, w)
    assert np.array_equal(y_fmt, y_ref)
    for which, (r, c) in [(0, (5, 100)), (1, (63, 0)), (2, (127, 63))]:
        assert oracle.blob_weight_fmt(H, I, FMT_INT4_G64, ex[1], which, r, c) == \
            oracle.blob_weight(H, I, ex[1], which, r, c)


@pytest.mark.parametrize("fmt,lo,hi", [(FMT_INT8_G64, -8, 7), (FMT_INT2_G64, -2, 1)])
def test_narrow_values_equal_int4(fmt, lo, hi):
    """int8 / int2 blobs holding int4-representable values give the int4 blob's y."""
    rng = np.random.default_rng(2 + fmt)
    parts = [rand_expert(rng, lo, hi, FMT_INT4_G64) for _ in range(E + 1)]
    y4 = layer([blob(FMT_INT4_G64, *p) for p in parts[:E]], blob(FMT_INT4_G64, *parts[E]),
               FMT_INT4_G64, *inputs(np.random.default_rng(9)))
    yf = layer([blob(fmt, *p) for p in parts[:E]], blob(fmt, *parts[E]), fmt, *inputs(np.random.default_rng(9)))
    assert np.array_equal(yf, y4)
    assert np.abs(y4).max() > 0


def test_int8_uses_all_eight_bits():
    """Values outside [-8, 7] change y (the codec is not a nibble decoder)."""
    rng = np.random.default_rng(5)
    parts = [rand_expert(rng, -8, 7, FMT_INT8_G64) for _ in range(E + 1)]
    y1 = layer([blob(FMT_INT8_G64, *p) for p in parts[:E]], blob(FMT_INT8_G64, *parts[E]),
               FMT_INT8_G64, *inputs(np.random.default_rng(9)))
    qg = parts[E][0].copy()
    qg[:, 3] = 100
    parts[E] = (qg,) + parts[E][1:]
    y2 = layer([blob(FMT_INT8_G64, *p) for p in parts[:E]], blob(FMT_INT8_G64, *parts[E]),
               FMT_INT8_G64, *inputs(np.random.default_rng(9)))
    assert not np.array_equal(y1, y2)


def test_per_row_equals_gs64_with_equal_group_scales():
    rng = np.random.default_rng(6)
    row_parts, g64_parts = [], []
    for _ in range(E + 1):
        qg, qu, qd, sg, su, sd = rand_expert(rng, -8, 7, FMT_INT4_ROW)
        row_parts.append((qg, qu, qd, sg, su, sd))
        g64_parts.append((qg, qu, qd, np.repeat(sg, H // 64, 1), np.repeat(su, H // 64, 1),
                          np.repeat(sd, I // 64, 1)))
    yr = layer([blob(FMT_INT4_ROW, *p) for p in row_parts[:E]], blob(FMT_INT4_ROW, *row_parts[E]),
               FMT_INT4_ROW, *inputs(np.random.default_rng(9)))
    yg = layer([blob(FMT_INT4_G64, *p) for p in g64_parts[:E]], blob(FMT_INT4_G64, *g64_parts[E]),
               FMT_INT4_G64, *inputs(np.random.default_rng(9)))
    assert np.array_equal(yr, yg)
    # and the row's scale is the one used: changing it for one row changes that column of y
    qg, qu, qd, sg, su, sd = row_parts[E]
    sd2 = sd.copy()
    sd2[7, 0] *= 2
    row_parts[E] = (qg, qu, qd, sg, su, sd2)
    yr2 = layer([blob(FMT_INT4_ROW, *p) for p in row_parts[:E]], blob(FMT_INT4_ROW, *row_parts[E]),
                FMT_INT4_ROW, *inputs(np.random.default_rng(9)))
    diff = np.nonzero((yr2 != yr).any(axis=0))[0]
    assert diff.tolist() == [7]


@pytest.mark.parametrize("fmt", [FMT_INT4_G64, FMT_INT8_G64, FMT_INT4_ROW, FMT_INT2_G64])
def test_quantizer_blob_decodes_to_its_dequantised_weights(fmt):
    """The package's host quantiser packs what the oracle's decoder reads back: every
    sampled weight of the blob equals the quantiser's dequantised value, and the rounding
    error is at most half a step (inside the code range)."""
    from int4_routed_expert_gemv_b200 import quantize as Q
    rng = np.random.default_rng(30 + fmt)
    G = (rng.standard_normal((I, H)) * 0.05).astype(np.float32)
    U = (rng.standard_normal((I, H)) * 0.05).astype(np.float32)
    D = (rng.standard_normal((H, I)) * 0.05).astype(np.float32)
    blob_q, (Gd, Ud, Dd) = Q.expert_blob(G, U, D, fmt)
    assert blob_q.size == oracle.blob_bytes_fmt(H, I, fmt)
    for which, M, Md in [(0, G, Gd), (1, U, Ud), (2, D, Dd)]:
        rows, cols = M.shape
        for r, c in zip(rng.integers(0, rows, 40), rng.integers(0, cols, 40)):
            assert oracle.blob_weight_fmt(H, I, fmt, blob_q, which, int(r), int(c)) == float(Md[r, c])
        q, s = Q.quantize_matrix(M, fmt)
        step = np.repeat(s.astype(np.float32), cols // s.shape[1], axis=1)
        lo, hi = Q.QRANGE[fmt]
        inside = (M / step > lo - 0.5) & (M / step < hi + 0.5)
        assert np.all(np.abs(M - Md)[inside] <= 0.5 * step[inside] * (1 + 1e-6))
