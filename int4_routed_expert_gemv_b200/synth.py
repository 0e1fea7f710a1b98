"""Seeded synthetic inputs for the routed int4 MoE layer.

This module only draws random numbers.  It holds none of the layer's arithmetic (no
dequantisation, no routing, no packing): the CUDA library and the CPU oracle both
receive exactly the arrays produced here.

Random sources
--------------
* Expert blobs (int4 nibbles and fp16 group scales) come from a counter-based hash
  (the splitmix64 output function of Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014), written with torch integer ops so the
  same bytes can be produced on the host or directly in device memory.  Any element can
  be regenerated on its own, which lets a checker rebuild only the experts it touches.
  Every byte value is a valid pair of int4 nibbles, so the nibble section is raw hash
  bytes: each nibble is uniform on [-8, 7] as a two's-complement value.
  Scales are ``fp16(0.005 + 0.015 * u)`` with ``u`` a 24-bit uniform on [0, 1), the two
  fp32 operations done one at a time and the result rounded to fp16 (nearest-even).
* Gaussian activations and router rows come from numpy's counter-based Philox generator
  on the host (float64 normals rounded to float32; bfloat16 activations are the float32
  values rounded to nearest-even by torch).
* The skewed-routing bias is ``b_e = -1.1 * ln(e + 1)``: the log of an unnormalised
  Zipf(s = 1.1) prior over expert rank e + 1.

Blob layout is the library's container layout: ``Gq [I][H/2] | Uq [I][H/2] | Dq [H][I/2]
| Gs [I][H/64] | Us [I][H/64] | Ds [H][I/64]`` (u8 nibbles, then fp16 scales).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

MASK64 = (1 << 64) - 1
GOLDEN = 0x9E3779B97F4A7C15
M1 = 0xBF58476D1CE4E5B9
M2 = 0x94D049BB133111EB
M3 = 0xD1B54A32D192ED03

# stream kinds for the hash generator
KIND_NIBBLES = 0
KIND_SCALES = 1
# stream kinds for the Philox generator
KIND_X = 1
KIND_WR = 2


def _s64(v: int) -> int:
    """Unsigned 64-bit value as the signed int64 with the same bits."""
    v &= MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def mix64_int(z: int) -> int:
    """splitmix64 output function on a Python int (mod 2^64)."""
    z &= MASK64
    z = ((z ^ (z >> 30)) * M1) & MASK64
    z = ((z ^ (z >> 27)) * M2) & MASK64
    return z ^ (z >> 31)


def _srl(z: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of int64 bits."""
    return (z >> s) & ((1 << (64 - s)) - 1)


def mix64(z: torch.Tensor) -> torch.Tensor:
    """splitmix64 output function on int64 tensors (two's-complement wrap-around)."""
    z = (z ^ _srl(z, 30)) * _s64(M1)
    z = (z ^ _srl(z, 27)) * _s64(M2)
    return z ^ _srl(z, 31)


def stream_key(seed: int, layer: int, tensor: int, kind: int) -> int:
    s0 = mix64_int(seed * GOLDEN + 1)
    sid = (layer << 24) | (tensor << 4) | kind
    return mix64_int(s0 ^ ((sid * M3) & MASK64))


def hash_words(key: int, start: int, count: int, device) -> torch.Tensor:
    """count 64-bit hash words (int64) for counters start .. start+count-1."""
    i = torch.arange(start + 1, start + count + 1, dtype=torch.int64, device=device)
    z = i * _s64(GOLDEN) + _s64(key)
    return mix64(z)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    hidden: int
    inter: int
    n_experts: int
    top_k: int
    n_shared: int = 1

    @property
    def blob_bytes(self) -> int:
        H, I = self.hidden, self.inter
        return 3 * (H * I // 2) + 2 * (I * (H // 64) * 2) + H * (I // 64) * 2

    @property
    def stride(self) -> int:
        """Expert blob stride: blob size rounded up to 256 bytes."""
        return (self.blob_bytes + 255) // 256 * 256


def expert_blob(shape: LayerShape, seed: int, layer: int, expert: int,
                device="cpu", out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """One expert's blob (uint8, shape.blob_bytes long).

    expert == shape.n_experts denotes the shared expert of that layer.
    """
    H, I = shape.hidden, shape.inter
    nib = 3 * (H * I // 2)
    n_scales = 2 * I * (H // 64) + H * (I // 64)
    if out is None:
        out = torch.empty(shape.blob_bytes, dtype=torch.uint8, device=device)
    assert out.numel() >= shape.blob_bytes and out.dtype == torch.uint8
    # nibble bytes: 8 bytes per hash word, little-endian byte order of the word
    kn = stream_key(seed, layer, expert, KIND_NIBBLES)
    nw = (nib + 7) // 8
    words = hash_words(kn, 0, nw, out.device)
    out[:nib].copy_(words.view(torch.uint8)[:nib])
    # fp16 scales: one hash word each, top 24 bits -> u in [0,1)
    ks = stream_key(seed, layer, expert, KIND_SCALES)
    w = hash_words(ks, 0, n_scales, out.device)
    u = _srl(w, 40).to(torch.float32) * (1.0 / 16777216.0)
    s32 = u * 0.015
    s32 = s32 + 0.005
    s16 = s32.to(torch.float16)
    out[nib:nib + 2 * n_scales].copy_(s16.view(torch.uint8))
    return out


def experts_tensor(shape: LayerShape, seed: int, layer: int = 0, device="cpu") -> torch.Tensor:
    """All routed experts of one layer, [E][stride] uint8 (padding bytes zero)."""
    buf = torch.zeros(shape.n_experts, shape.stride, dtype=torch.uint8, device=device)
    for e in range(shape.n_experts):
        expert_blob(shape, seed, layer, e, out=buf[e, :shape.blob_bytes])
    return buf


def shared_tensor(shape: LayerShape, seed: int, layer: int = 0, device="cpu") -> torch.Tensor:
    buf = torch.zeros(shape.stride, dtype=torch.uint8, device=device)
    expert_blob(shape, seed, layer, shape.n_experts, out=buf[:shape.blob_bytes])
    return buf


def _philox(seed: int, layer: int, kind: int, variant: int) -> np.random.Generator:
    key = (seed << 64) | (layer << 32) | (kind << 16) | variant
    return np.random.Generator(np.random.Philox(key=key))


def normal_f32(seed: int, layer: int, kind: int, variant: int, shape, std: float = 1.0) -> np.ndarray:
    g = _philox(seed, layer, kind, variant)
    v = g.standard_normal(size=shape, dtype=np.float64)
    if std != 1.0:
        v = v * std
    return v.astype(np.float32)


def router_weight(shape: LayerShape, seed: int, layer: int = 0) -> np.ndarray:
    """W_r [E][H] float32, N(0, 0.02^2)."""
    return normal_f32(seed, layer, KIND_WR, 0, (shape.n_experts, shape.hidden), std=0.02)


def activations(shape: LayerShape, seed: int, tokens: int, variant: int = 0,
                layer: int = 0) -> np.ndarray:
    """x [T][H] float32, N(0, 1)."""
    return normal_f32(seed, layer, KIND_X, variant, (tokens, shape.hidden))


def activations_bf16(shape: LayerShape, seed: int, tokens: int, variant: int = 0) -> torch.Tensor:
    """x [T][H] bfloat16 (float32 normals rounded to nearest-even)."""
    return torch.from_numpy(activations(shape, seed, tokens, variant)).to(torch.bfloat16)


def zipf_bias(n_experts: int, s: float = 1.1) -> np.ndarray:
    """b_e = -s * ln(e + 1), float32."""
    e = np.arange(n_experts, dtype=np.float64)
    return (-s * np.log(e + 1.0)).astype(np.float32)


# ------------------------------------------------------------------------------------
# Named workloads
# ------------------------------------------------------------------------------------

@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    tokens: int
    seed: int
    x_variant: int
    zipf: bool = False
    x_dtype: str = "f32"      # "f32" or "bf16"
    layers: int = 1
    description: str = ""


SMALL = LayerShape(hidden=1024, inter=512, n_experts=64, top_k=4, n_shared=1)
GLM = LayerShape(hidden=6144, inter=2048, n_experts=256, top_k=8, n_shared=1)

WORKLOADS = {
    w.name: w for w in [
        Workload("moe_h1024_i512_e64_k4_t1", SMALL, 1, seed=0, x_variant=0,
                 description="one MoE layer, hidden 1024, 64 experts of intermediate 512, "
                             "top-4 + 1 shared, 1 token, fp32"),
        Workload("glm52_moe_h6144_i2048_e256_k8_t1", GLM, 1, seed=1, x_variant=0,
                 description="GLM-5.2-shaped MoE layer decode: hidden 6144, 256 experts of "
                             "intermediate 2048, top-8 + 1 shared, 1 token, fp32"),
        Workload("glm52_moe_h6144_i2048_e256_k8_t4_zipf", GLM, 4, seed=1, x_variant=1,
                 zipf=True,
                 description="GLM-5.2-shaped layer, 4-token verify batch, Zipf(1.1) router bias"),
        Workload("moe_h1024_i512_e64_k4_t4_zipf", SMALL, 4, seed=0, x_variant=1, zipf=True,
                 description="hidden-1024 layer, 4-token verify batch, Zipf(1.1) router bias"),
        Workload("glm52_stack16_h6144_i2048_e256_k8_t1", GLM, 1, seed=3, x_variant=0,
                 layers=16,
                 description="16 GLM-5.2-shaped layers, x <- x + MoE(RMSNorm(x)), 1 token"),
        Workload("moe_h1024_i512_e64_k4_stack16_t1", SMALL, 1, seed=3, x_variant=0, layers=16,
                 description="16 hidden-1024 layers (64 experts of intermediate 512, top-4 + 1 "
                             "shared each), x <- x + MoE(RMSNorm(x)), 1 token"),
        Workload("moe_h1024_i512_e64_k4_t2048_bf16_zipf", SMALL, 2048, seed=0, x_variant=2,
                 zipf=True, x_dtype="bf16",
                 description="prefill-like 2048 bf16 tokens through the hidden-1024 layer, "
                             "Zipf(1.1) routing, grouped tensor-core GEMM"),
        Workload("glm52_moe_h6144_i2048_e256_k8_t2048_bf16_zipf", GLM, 2048, seed=1,
                 x_variant=2, zipf=True, x_dtype="bf16",
                 description="prefill-like 2048 bf16 tokens through the GLM-5.2-shaped layer, "
                             "Zipf(1.1) routing, grouped tensor-core GEMM"),
    ]
}
