"""Pins of the oracle's two Python composition helpers (CPU only).

  * oracle.forward_sparse packs the selected experts' blobs into a compact array and
    renumbers idx into it.  It must give exactly the result of oracle.forward on the full
    expert array (the C function, pinned in test_oracle.py), whatever extra experts the
    dict holds and in whatever order the ids come.
  * oracle.stack_layer is one residual layer: n = RMSNorm(x), routing on n, the MoE
    forward on n, x + y in float32.  It must equal that composition written out here from
    the pinned C primitives (rmsnorm, route, the full-array forward), and it must not equal
    the compositions a slip would give (routing on x instead of n, no residual).
"""
import numpy as np
import pytest

import oracle
from int4_routed_expert_gemv_b200 import synth

SHAPE = synth.LayerShape(hidden=128, inter=64, n_experts=8, top_k=3, n_shared=1)
SEED = 11


def _layer(shape=SHAPE, seed=SEED):
    experts = synth.experts_tensor(shape, seed).numpy()
    shared = synth.shared_tensor(shape, seed).numpy()
    wr = synth.router_weight(shape, seed) * 5.0   # wide logit spread: no near-ties
    return experts, shared, wr


@pytest.mark.parametrize("T", [1, 3, 7])
def test_forward_sparse_equals_full_forward(T):
    s = SHAPE
    experts, shared, wr = _layer()
    x = synth.activations(s, SEED, T, variant=T)
    idx, w, _ = oracle.route(x, wr, None, s.top_k)
    full = oracle.forward(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared, x, experts, s.stride,
                          shared, idx, w)
    used = sorted({int(e) for e in idx.ravel()})
    blobs = {e: experts[e, :s.blob_bytes] for e in used}
    sparse = oracle.forward_sparse(s.hidden, s.inter, s.top_k, s.n_shared, x, blobs, shared, idx, w)
    assert np.array_equal(sparse, full)
    # extra, unselected experts in the dict, inserted in descending id order
    blobs_all = {e: experts[e, :s.blob_bytes] for e in reversed(range(s.n_experts))}
    sparse2 = oracle.forward_sparse(s.hidden, s.inter, s.top_k, s.n_shared, x, blobs_all, shared, idx, w)
    assert np.array_equal(sparse2, full)


def test_forward_sparse_uses_the_expert_it_is_given():
    """A dict whose blob for one selected id is another expert's blob changes y: the
    renumbering reaches the blob that belongs to the id."""
    s = SHAPE
    experts, shared, wr = _layer()
    x = synth.activations(s, SEED, 2, variant=5)
    idx, w, _ = oracle.route(x, wr, None, s.top_k)
    used = sorted({int(e) for e in idx.ravel()})
    blobs = {e: experts[e, :s.blob_bytes] for e in used}
    good = oracle.forward_sparse(s.hidden, s.inter, s.top_k, s.n_shared, x, blobs, shared, idx, w)
    other = next(e for e in range(s.n_experts) if e not in used)
    blobs[used[0]] = experts[other, :s.blob_bytes]
    bad = oracle.forward_sparse(s.hidden, s.inter, s.top_k, s.n_shared, x, blobs, shared, idx, w)
    assert not np.array_equal(good, bad)


@pytest.mark.parametrize("T", [1, 4])
def test_stack_layer_equals_hand_composition(T):
    s = SHAPE
    experts, shared, wr = _layer()
    x = synth.activations(s, SEED, T, variant=20 + T) * 3.0
    gamma = (0.5 + np.arange(s.hidden, dtype=np.float32) / s.hidden).astype(np.float32)
    eps = 1e-5

    x_out, n, idx, w, logits, y = oracle.stack_layer(
        x, gamma, eps, wr, None, s.top_k, s.hidden, s.inter, s.n_shared,
        lambda e: experts[e, :s.blob_bytes], shared)

    # the composition written out from the pinned primitives
    n_ref = oracle.rmsnorm(x, gamma, eps)
    idx_ref, w_ref, logits_ref = oracle.route(n_ref, wr, None, s.top_k)
    y_ref = oracle.forward(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared, n_ref, experts, s.stride,
                           shared, idx_ref, w_ref)
    x_ref = (x.astype(np.float32) + y_ref.astype(np.float32)).astype(np.float32)

    assert np.array_equal(n, n_ref)
    assert np.array_equal(idx, idx_ref) and np.array_equal(w, w_ref) and np.array_equal(logits, logits_ref)
    assert np.array_equal(y, y_ref)
    assert x_out.dtype == np.float32 and np.array_equal(x_out, x_ref)

    # the slips the helper must not make: routing on x, forwarding x, dropping the residual
    idx_x, w_x, _ = oracle.route(x, wr, None, s.top_k)
    y_on_x = oracle.forward(s.hidden, s.inter, s.n_experts, s.top_k, s.n_shared, x, experts, s.stride,
                            shared, idx_x, w_x)
    assert not np.array_equal(y, y_on_x)
    assert not np.array_equal(x_out, y_ref)


def test_rmsnorm_scales_by_gamma():
    """RMSNorm's gamma multiplies per column (a transposed or dropped gamma shows)."""
    s = SHAPE
    x = synth.activations(s, SEED, 2, variant=40)
    g1 = np.ones(s.hidden, np.float32)
    g2 = np.full(s.hidden, 2.0, np.float32)
    n1 = oracle.rmsnorm(x, g1, 1e-5)
    n2 = oracle.rmsnorm(x, g2, 1e-5)
    assert np.array_equal(n2, (n1.astype(np.float64) * 2.0).astype(np.float32))
    rms = np.sqrt(np.mean(n1.astype(np.float64) ** 2, axis=1))
    assert np.allclose(rms, 1.0, rtol=1e-5)
