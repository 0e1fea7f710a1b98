"""Pins for the CPU oracle: checks against things other than the oracle itself.

The pages print no worked example of the layer, so the oracle is pinned by
  * exhaustive encodings (all 256 bytes, all 65536 fp16 patterns) against independent
    decoders (int8 arithmetic shifts, numpy's float16),
  * pack -> oracle-unpack round trips through a packer written here from the container
    description (low nibble first, fp16 scale per 64 input columns),
  * closed forms (constant-weight layer, golden file), zero input, RMSNorm of a constant,
  * special cases that reduce to library routines: all experts selected -> dense softmax
    mixture (numpy matmul + scipy softmax/expit), routing against a stable numpy argsort,
    union against np.unique / stable argsort,
  * brute force dense-then-mask evaluation on tiny layers,
  * invariants (weights sum to 1, non-increasing, union sorted and complete).
"""
import math
import os

import numpy as np
import pytest
import scipy.special as sp
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------
# an independent packer, written from the container description
# ------------------------------------------------------------------------------------

def pack_rows(q: np.ndarray) -> np.ndarray:
    """q [rows][cols] ints in [-8,7] -> [rows][cols/2] bytes, column 2j in the low nibble."""
    u = (q.astype(np.int64) & 0xF).astype(np.uint8)
    return (u[:, 0::2] | (u[:, 1::2] << 4)).astype(np.uint8)


def make_blob(qg, sg, qu, su, qd, sd) -> np.ndarray:
    """Blob = Gq | Uq | Dq | Gs | Us | Ds (scales as float16 arrays)."""
    parts = [pack_rows(qg).ravel(), pack_rows(qu).ravel(), pack_rows(qd).ravel(),
             sg.astype(np.float16).view(np.uint8).ravel(),
             su.astype(np.float16).view(np.uint8).ravel(),
             sd.astype(np.float16).view(np.uint8).ravel()]
    return np.concatenate(parts)


def random_expert(rng, H, I, smin=0.005, smax=0.02):
    qg = rng.integers(-8, 8, (I, H))
    qu = rng.integers(-8, 8, (I, H))
    qd = rng.integers(-8, 8, (H, I))
    sg = rng.uniform(smin, smax, (I, H // 64)).astype(np.float16)
    su = rng.uniform(smin, smax, (I, H // 64)).astype(np.float16)
    sd = rng.uniform(smin, smax, (H, I // 64)).astype(np.float16)
    dense = dict(G=qg * np.repeat(sg.astype(np.float64), 64, axis=1),
                 U=qu * np.repeat(su.astype(np.float64), 64, axis=1),
                 D=qd * np.repeat(sd.astype(np.float64), 64, axis=1))
    return make_blob(qg, sg, qu, su, qd, sd), dense


def dense_expert(dense, x64):
    g = dense["G"] @ x64
    u = dense["U"] @ x64
    h = g * sp.expit(g) * u
    return dense["D"] @ h


# ------------------------------------------------------------------------------------
# encodings
# ------------------------------------------------------------------------------------

def test_nibble_all_bytes():
    for b in range(256):
        row = np.array([b], np.uint8)
        lo = np.int8(np.uint8((b << 4) & 0xFF).view(np.int8)) >> 4   # arithmetic shift
        hi = np.uint8(b).view(np.int8) >> 4
        assert oracle.nibble(row, 0) == int(lo), b
        assert oracle.nibble(row, 1) == int(hi), b
    vals = {oracle.nibble(np.array([b], np.uint8), 0) for b in range(16)}
    assert vals == set(range(-8, 8))


def test_half_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    for b in range(0, 65536, 1):
        v = oracle.half(int(b))
        r = ref[b]
        if math.isnan(r):
            assert math.isnan(v)
        else:
            assert v == r and math.copysign(1, v) == math.copysign(1, r), b


def test_bf16_round_golden_and_torch():
    # ties to even around 1.0 (bf16 spacing at 1 is 2^-7)
    assert oracle.bf16_round(1.0 + 2 ** -8) == 1.0
    assert oracle.bf16_round(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6
    assert oracle.bf16_round(1.0 + 2 ** -8 + 2 ** -20) == 1.0 + 2 ** -7
    assert oracle.bf16_round(-1.0 - 2 ** -8) == -1.0
    rng = np.random.default_rng(5)
    v = rng.standard_normal(4000).astype(np.float32) * np.float32(10.0) ** rng.integers(-6, 6, 4000)
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float32).numpy()
    got = np.array([oracle.bf16_round(float(a)) for a in v], np.float32)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("H,I", [(64, 64), (128, 192), (256, 64)])
def test_blob_roundtrip(H, I):
    rng = np.random.default_rng(H * 7 + I)
    blob, dense = random_expert(rng, H, I)
    assert len(blob) == oracle.blob_bytes(H, I)
    for which, name, rows, cols in [(0, "G", I, H), (1, "U", I, H), (2, "D", H, I)]:
        M = dense[name]
        rr = rng.integers(0, rows, 40).tolist() + [0, rows - 1]
        cc = rng.integers(0, cols, 40).tolist() + [0, 63, 64 % cols, cols - 1]
        for r in rr:
            for c in cc:
                assert oracle.blob_weight(H, I, blob, which, r, c) == M[r, c], (name, r, c)


def test_bytes_per_expert():
    # 3 int4 matrices of H*I plus one fp16 scale per 64 weights: 1.59375 bytes/(H*I)
    assert oracle.blob_bytes(6144, 2048) == 20054016
    assert oracle.blob_bytes(1024, 512) == 835584
    assert oracle.blob_bytes(6144, 2048) == int(1.59375 * 6144 * 2048)


# ------------------------------------------------------------------------------------
# expert FFN and forward
# ------------------------------------------------------------------------------------

def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                k, v = line.split("=", 1)
                vals[k.strip()] = v.strip()
    return vals


def test_closed_form_constant_layer_golden():
    g = _read_golden("const_layer.txt")
    H, I = int(g["H"]), int(g["I"])
    qg, qu, qd = int(g["q_gate"]), int(g["q_up"]), int(g["q_down"])
    sg, su, sd = float(g["s_gate"]), float(g["s_up"]), float(g["s_down"])
    xv = float(g["x"])
    blob = make_blob(np.full((I, H), qg), np.full((I, H // 64), sg, np.float16),
                     np.full((I, H), qu), np.full((I, H // 64), su, np.float16),
                     np.full((H, I), qd), np.full((H, I // 64), sd, np.float16))
    x = np.full((1, H), xv, np.float32)
    out, h = oracle.expert(H, I, blob, x[0])
    exp_h = float(g["h"])
    exp_expert = float(g["expert_out"])
    assert np.allclose(h, exp_h, rtol=1e-15, atol=0)
    assert np.allclose(out, exp_expert, rtol=1e-15, atol=0)
    # layer: shared + two routed copies with weights w and 1-w
    E = 2
    experts = np.stack([blob, blob])
    idx = np.array([[1, 0]], np.int32)
    w = np.array([[0.75, 0.25]], np.float32)
    y = oracle.forward(H, I, E, 2, 1, x, experts, len(blob), blob, idx, w)
    assert np.allclose(y, np.float32(float(g["layer_out"])), rtol=0, atol=0)


def test_gate_up_not_interchangeable():
    # silu(g)*u != silu(u)*g for g != u: swapping gate and up must change the result
    H = I = 64
    mk = lambda qa, qb: make_blob(np.full((I, H), qa), np.full((I, 1), 0.25, np.float16),
                                  np.full((I, H), qb), np.full((I, 1), 0.25, np.float16),
                                  np.full((H, I), 1), np.full((H, 1), 0.25, np.float16))
    x = np.full(H, 0.125, np.float32)
    a, _ = oracle.expert(H, I, mk(1, 3), x)
    b, _ = oracle.expert(H, I, mk(3, 1), x)
    g, u = 64 * 0.25 * 0.125, 3 * 64 * 0.25 * 0.125
    assert np.allclose(a, 64 * 0.25 * (g * sp.expit(g) * u), rtol=1e-14)
    assert np.allclose(b, 64 * 0.25 * (u * sp.expit(u) * g), rtol=1e-14)
    assert not np.allclose(a, b)


@pytest.mark.parametrize("H,I", [(64, 64), (128, 64), (64, 192)])
def test_expert_matches_dense_numpy(H, I):
    rng = np.random.default_rng(H + 3 * I)
    blob, dense = random_expert(rng, H, I)
    for _ in range(3):
        x = rng.standard_normal(H).astype(np.float32)
        out, _ = oracle.expert(H, I, blob, x)
        ref = dense_expert(dense, x.astype(np.float64))
        assert np.allclose(out, ref, rtol=1e-12, atol=1e-14 * np.abs(ref).max())


def _tiny_layer(rng, H, I, E):
    blobs, denses = [], []
    for _ in range(E + 1):
        b, d = random_expert(rng, H, I)
        blobs.append(b)
        denses.append(d)
    stride = len(blobs[0])
    return np.stack(blobs[:E]), blobs[E], stride, denses[:E], denses[E]


@pytest.mark.parametrize("E,k", [(4, 1), (4, 2), (6, 3), (8, 8), (5, 5)])
def test_forward_dense_then_mask(E, k):
    rng = np.random.default_rng(100 * E + k)
    H, I, T = 64, 128, 3
    experts, shared, stride, dense, dshared = _tiny_layer(rng, H, I, E)
    x = rng.standard_normal((T, H)).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.3).astype(np.float32)
    idx, w, logits = oracle.route(x, wr, None, k)
    y = oracle.forward(H, I, E, k, 1, x, experts, stride, shared, idx, w)
    for t in range(T):
        x64 = x[t].astype(np.float64)
        all_out = np.stack([dense_expert(d, x64) for d in dense])        # dense: every expert
        mask = np.zeros(E)
        mask[idx[t]] = w[t].astype(np.float64)                            # then mask
        ref = dense_expert(dshared, x64) + mask @ all_out
        assert np.allclose(y[t], ref, rtol=2e-7, atol=2e-7 * np.abs(ref).max())
        if k == E:
            # every expert selected: the routed part is the full softmax mixture
            p = sp.softmax(logits[t].astype(np.float64))
            ref2 = dense_expert(dshared, x64) + p @ all_out
            assert np.allclose(y[t], ref2, rtol=1e-6, atol=1e-6 * np.abs(ref2).max())


def test_zero_input_gives_zero_output():
    rng = np.random.default_rng(1)
    H, I, E, k = 64, 64, 4, 2
    experts, shared, stride, _, _ = _tiny_layer(rng, H, I, E)
    x = np.zeros((2, H), np.float32)
    wr = rng.standard_normal((E, H)).astype(np.float32)
    out = oracle.layer(H, I, E, k, 1, x, wr, None, experts, stride, shared)
    assert np.array_equal(out["y"], np.zeros((2, H), np.float32))
    # all logits zero -> experts 0..k-1 chosen with weight 1/k
    assert out["idx"].tolist() == [[0, 1], [0, 1]]
    assert np.all(out["w"] == np.float32(0.5))


def test_shared_only_when_routed_weights_zero():
    rng = np.random.default_rng(2)
    H, I, E, k = 64, 64, 4, 2
    experts, shared, stride, dense, dshared = _tiny_layer(rng, H, I, E)
    x = rng.standard_normal((1, H)).astype(np.float32)
    y = oracle.forward(H, I, E, k, 1, x, experts, stride, shared,
                       np.array([[0, 1]], np.int32), np.zeros((1, 2), np.float32))
    ref = dense_expert(dshared, x[0].astype(np.float64))
    assert np.allclose(y[0], ref, rtol=1e-6, atol=1e-7 * np.abs(ref).max())
    # without the shared expert the same call gives exactly zero
    y0 = oracle.forward(H, I, E, k, 0, x, experts, stride, None,
                        np.array([[0, 1]], np.int32), np.zeros((1, 2), np.float32))
    assert np.array_equal(y0, np.zeros_like(y0))


def test_bf16_mode_exact_when_representable():
    # power-of-two scales and |q| <= 8 make q*s exact in bf16; h rounding is then the
    # only difference, reproduced here with torch's bf16 conversion
    H = I = 64
    rng = np.random.default_rng(3)
    q = [rng.integers(-8, 8, s) for s in [(I, H), (I, H), (H, I)]]
    s = [np.full((I, 1), 2.0 ** -6, np.float16), np.full((I, 1), 2.0 ** -5, np.float16),
         np.full((H, 1), 2.0 ** -7, np.float16)]
    blob = make_blob(q[0], s[0], q[1], s[1], q[2], s[2])
    x = torch.from_numpy(rng.standard_normal(H).astype(np.float32)).to(torch.bfloat16).float().numpy()
    out32, h32 = oracle.expert(H, I, blob, x, bf16=False)
    out16, h16 = oracle.expert(H, I, blob, x, bf16=True)
    h_ref = torch.from_numpy(h32.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.array_equal(h16, h_ref)
    D = q[2] * 2.0 ** -7
    assert np.allclose(out16, D @ h_ref, rtol=1e-14, atol=1e-14)


def test_bf16_mode_rounds_weights():
    # a scale whose product with q is not a bf16 value: bf16 mode must use the rounded
    # weight (torch conversion), fp32 mode the exact one
    H = I = 64
    sc = np.float16(0.0131)                        # 11-bit mantissa
    qg = np.full((I, H), 7)
    blob = make_blob(qg, np.full((I, 1), sc, np.float16), qg, np.full((I, 1), sc, np.float16),
                     np.full((H, I), 1), np.full((H, 1), 2.0 ** -4, np.float16))
    wexact = 7 * float(sc)
    wb = float(torch.tensor(wexact, dtype=torch.float32).to(torch.bfloat16).float())
    assert wb != wexact
    assert oracle.blob_weight(H, I, blob, 0, 3, 5, bf16=False) == wexact
    assert oracle.blob_weight(H, I, blob, 0, 3, 5, bf16=True) == wb


# ------------------------------------------------------------------------------------
# routing
# ------------------------------------------------------------------------------------

def test_route_zero_router_and_bias_only():
    E, H, k = 16, 64, 5
    x = np.random.default_rng(0).standard_normal((3, H)).astype(np.float32)
    idx, w, _ = oracle.route(x, np.zeros((E, H), np.float32), None, k)
    assert idx.tolist() == [list(range(k))] * 3
    assert np.all(w == np.float32(1.0 / k))
    b = np.array([0.5, 2.0, -1.0, 2.0, 0.25, 3.0, -7, 0.5, 1.0, 1.5, 2.0, 0, 0, 0, 0, 9.0],
                 np.float32)
    idx, w, lg = oracle.route(x, np.zeros((E, H), np.float32), b, k)
    order = np.argsort(-b.astype(np.float64), kind="stable")[:k]
    assert idx.tolist() == [order.tolist()] * 3 == [[15, 5, 1, 3, 10]] * 3
    ref = sp.softmax(b[order].astype(np.float64))
    assert np.allclose(w, ref.astype(np.float32), rtol=0, atol=1e-7)


def test_route_duplicate_rows_lower_index_wins():
    rng = np.random.default_rng(4)
    E, H, k = 8, 128, 3
    wr = rng.standard_normal((E, H)).astype(np.float32)
    x = rng.standard_normal((1, H)).astype(np.float32)
    _, _, lg = oracle.route(x, wr, None, 1)
    best = int(np.argmax(lg[0]))
    wr2 = np.concatenate([wr, wr[best:best + 1]])       # the copy gets a higher index
    idx, w, lg2 = oracle.route(x, wr2, None, k)
    assert idx[0, 0] == best and lg2[0, E] == lg2[0, best]
    assert idx[0, 1] == E
    assert w[0, 0] == w[0, 1]
    wr3 = np.concatenate([wr[best:best + 1], wr])       # now the copy has the lower index
    idx3, _, _ = oracle.route(x, wr3, None, k)
    assert idx3[0, 0] == 0 and idx3[0, 1] == best + 1


@pytest.mark.parametrize("E,H,k,T", [(64, 1024, 4, 5), (256, 512, 8, 3), (7, 64, 7, 2)])
def test_route_against_numpy(E, H, k, T):
    rng = np.random.default_rng(E + H + k)
    x = rng.standard_normal((T, H)).astype(np.float32)
    wr = (rng.standard_normal((E, H)) * 0.02).astype(np.float32)
    b = (rng.standard_normal(E) * 0.1).astype(np.float32)
    idx, w, lg = oracle.route(x, wr, b, k)
    ref = (x.astype(np.float64) @ wr.astype(np.float64).T + b.astype(np.float64)).astype(np.float32)
    # same double-precision sum in another order: equal floats, or one ulp apart at most
    assert np.all(np.abs(lg.view(np.int32) - ref.view(np.int32)) <= 1)
    for t in range(T):
        order = np.argsort(-lg[t].astype(np.float64), kind="stable")[:k]
        assert idx[t].tolist() == order.tolist()
        p = sp.softmax(lg[t].astype(np.float64))
        assert np.allclose(w[t], p[order] / p[order].sum(), rtol=0, atol=1e-7)
        assert abs(float(w[t].astype(np.float64).sum()) - 1.0) <= 1e-6
        assert np.all(np.diff(w[t]) <= 0)


def test_route_rejects_non_finite():
    x = np.ones((1, 64), np.float32)
    wr = np.ones((4, 64), np.float32)
    x[0, 3] = np.nan
    with pytest.raises(oracle.OracleError):
        oracle.route(x, wr, None, 2)
    x[0, 3] = 1.0
    wr[2, 5] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.route(x, wr, None, 2)
    with pytest.raises(oracle.OracleError):
        oracle.route(np.ones((1, 64), np.float32), np.ones((4, 64), np.float32), None, 5)


# ------------------------------------------------------------------------------------
# union
# ------------------------------------------------------------------------------------

@pytest.mark.parametrize("E,k,T", [(8, 2, 1), (64, 4, 4), (256, 8, 37), (16, 16, 3), (32, 1, 0)])
def test_union_against_numpy(E, k, T):
    rng = np.random.default_rng(E * 31 + k * 7 + T)
    idx = np.array([rng.permutation(E)[:k] for _ in range(T)], np.int32).reshape(T, k)
    uid, nu, off, asg = oracle.union(idx, E)
    flat = idx.ravel()
    uniq = np.unique(flat)
    assert nu == len(uniq)
    assert uid[:nu].tolist() == uniq.tolist() and np.all(uid[nu:] == -1)
    order = np.argsort(flat, kind="stable")             # positions grouped by expert, ascending
    assert asg.tolist() == order.tolist()
    counts = np.array([np.sum(flat == e) for e in uniq])
    assert off[:nu].tolist() == (np.cumsum(counts) - counts).tolist()
    assert np.all(off[nu:] == T * k)
    # invariants: every (t, slot) exactly once; union no larger than min(E, T*k)
    assert sorted(asg.tolist()) == list(range(T * k))
    assert nu <= min(E, T * k)
    for u in range(nu):
        seg = asg[off[u]:(off[u + 1] if u + 1 < nu else T * k)]
        assert np.all(flat[seg] == uid[u]) and np.all(np.diff(seg) > 0)


def test_union_rejects_bad_ids():
    with pytest.raises(oracle.OracleError):
        oracle.union(np.array([[1, 1]], np.int32), 4)
    with pytest.raises(oracle.OracleError):
        oracle.union(np.array([[0, 4]], np.int32), 4)
    with pytest.raises(oracle.OracleError):
        oracle.union(np.array([[-1, 2]], np.int32), 4)


# ------------------------------------------------------------------------------------
# RMSNorm
# ------------------------------------------------------------------------------------

def test_rmsnorm_closed_form_and_numpy():
    H = 128
    for c in [1.0, -3.5, 1e-3]:
        x = np.full((1, H), c, np.float32)
        out = oracle.rmsnorm(x, np.ones(H, np.float32), 1e-5)
        ref = np.float32(c / math.sqrt(c * c + 1e-5))
        assert np.all(np.abs(out - ref) <= np.abs(ref) * 2 ** -23)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((4, H)).astype(np.float32)
    gmm = rng.uniform(0.5, 1.5, H).astype(np.float32)
    out = oracle.rmsnorm(x, gmm, 1e-5)
    x64 = x.astype(np.float64)
    ref = x64 / np.sqrt(np.mean(x64 ** 2, axis=1, keepdims=True) + 1e-5) * gmm
    assert np.allclose(out, ref, rtol=2 ** -23, atol=0)


def test_bf16_weights_exact_h_mode():
    # mode 2 rounds only the weights: with bf16-representable weights it equals the fp32
    # contract exactly, and it differs from mode 1 exactly by the rounding of h
    H = I = 64
    rng = np.random.default_rng(11)
    q = [rng.integers(-8, 8, s) for s in [(I, H), (I, H), (H, I)]]
    s = [np.full((I, 1), 2.0 ** -6, np.float16), np.full((I, 1), 2.0 ** -5, np.float16),
         np.full((H, 1), 2.0 ** -7, np.float16)]
    blob = make_blob(q[0], s[0], q[1], s[1], q[2], s[2])
    x = torch.from_numpy(rng.standard_normal(H).astype(np.float32)).to(torch.bfloat16).float().numpy()
    out0, h0 = oracle.expert(H, I, blob, x, bf16=0)
    out2, h2 = oracle.expert(H, I, blob, x, bf16=2)
    out1, h1 = oracle.expert(H, I, blob, x, bf16=1)
    assert np.array_equal(out0, out2) and np.array_equal(h0, h2)
    assert not np.array_equal(h1, h2)
    assert np.array_equal(h1, torch.from_numpy(h2.astype(np.float32)).to(torch.bfloat16).double().numpy())
    # non-representable weights: mode 2 uses the rounded weights, like mode 1
    blob, dense = random_expert(rng, H, I)
    for r, c in [(0, 0), (5, 63), (63, 1)]:
        assert (oracle.blob_weight(H, I, blob, 0, r, c, bf16=2) ==
                oracle.blob_weight(H, I, blob, 0, r, c, bf16=1))
