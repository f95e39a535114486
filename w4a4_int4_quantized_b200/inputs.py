"""Seeded synthetic inputs for the W4A4 ConvRot linear layer.

This module holds no arithmetic of the method: it only draws random numbers
(NumPy PCG64, ``default_rng(seed)``), shapes them like the Flux-class DiT
layers the pages run (hidden size 3072, MLP 12288, 4096 image + 512 text
tokens), plants outlier channels, and narrows fp32 draws to bf16 with
round-to-nearest-even.  Both the CUDA path and the CPU oracle consume exactly
these arrays; bf16 tensors are returned as uint16 bit patterns.

Workloads (the pages measure only end-to-end image generation with Krea 2
Turbo, whose weights are not available; these stand in for its layers):
  * ``tiny``        X[64,256] N(0,1) with channels {5,70,135,200} x100,
                    W[256,256] N(0,0.02), group 64, rank 16 (L1, L2 N(0,0.01)),
                    zero bias.
  * ``attn_proj``   X[4608,3072] N(0,1) with 1% of channels (31, drawn without
                    replacement) scaled by U[50,200], W[3072,3072] N(0,0.02),
                    group 128, no low-rank, bias N(0,0.01).
  * ``mlp_up`` / ``mlp_down``  3072->12288 and 12288->3072 at M=4608, group 128,
                    rank 128.
  * ``qkv``/``out``/``first``/``last``/``tmlp``: the double-stream block at
                    M=9216 (W4A4 rank 64 and W8A8 group 128).
  * ``sweep``       M x (K,N) x rank points with 1% x100 outliers.
Outlier channels follow "ComfyUI-INT4-Fast" (kongchang.com, "INT4 Quantized
Inference Comes to ComfyUI"): a few channels with magnitudes 100x the rest.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Narrow fp32 to bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


@dataclass
class LayerSpec:
    name: str
    M: int
    K: int
    N: int
    group: int
    rank: int = 0
    bias: bool = True
    w8a8: bool = False
    seed: int = 0
    outlier_channels: tuple | None = None   # fixed channel list, scaled by outlier_scale
    outlier_frac: float = 0.01              # else round(frac*K) channels drawn by rng.choice
    outlier_lo: float = 50.0
    outlier_hi: float = 200.0
    outlier_scale: float | None = None      # fixed scale (tiny / sweep); else U[lo,hi]
    w_std: float = 0.02
    lr_std: float = 0.01
    b_std: float = 0.01
    extra: dict = field(default_factory=dict)


WORKLOADS: dict[str, LayerSpec] = {
    "tiny": LayerSpec("tiny", 64, 256, 256, 64, rank=16, bias=False, seed=0,
                      outlier_channels=(5, 70, 135, 200), outlier_scale=100.0),
    "attn_proj": LayerSpec("attn_proj", 4608, 3072, 3072, 128, rank=0, bias=True, seed=2),
    "mlp_up": LayerSpec("mlp_up", 4608, 3072, 12288, 128, rank=128, bias=True, seed=3),
    "mlp_down": LayerSpec("mlp_down", 4608, 12288, 3072, 128, rank=128, bias=True, seed=3),
    "block_qkv": LayerSpec("block_qkv", 9216, 3072, 9216, 128, rank=64, seed=4),
    "block_out": LayerSpec("block_out", 9216, 3072, 3072, 128, rank=64, seed=4),
    "block_mlp_up": LayerSpec("block_mlp_up", 9216, 3072, 12288, 128, rank=64, seed=4),
    "block_mlp_down": LayerSpec("block_mlp_down", 9216, 12288, 3072, 128, rank=64, seed=4),
    "block_first_w8a8": LayerSpec("block_first_w8a8", 9216, 3072, 3072, 128, w8a8=True, seed=4),
    "block_last_w8a8": LayerSpec("block_last_w8a8", 9216, 3072, 3072, 128, w8a8=True, seed=4),
    "block_tmlp_w8a8": LayerSpec("block_tmlp_w8a8", 2, 256, 3072, 128, w8a8=True, seed=4),
    # a point of the shape sweep: the MLP down-projection shape at 256 tokens,
    # too few tiles for the persistent GEMM (it runs in the split-K form)
    "m256_down": LayerSpec("m256_down", 256, 12288, 3072, 128, rank=0, bias=True, seed=1043,
                           outlier_scale=100.0),
}


def sweep_spec(index: int, M: int, K: int, N: int, rank: int) -> LayerSpec:
    return LayerSpec(f"sweep{index}", M, K, N, 128, rank=rank, seed=1000 + index,
                     outlier_scale=100.0)


def make_activations(spec: LayerSpec, rng: np.random.Generator, M: int | None = None) -> np.ndarray:
    M = spec.M if M is None else M
    X = rng.standard_normal((M, spec.K), dtype=np.float32)
    if spec.outlier_channels is not None:
        ch = np.asarray(spec.outlier_channels, dtype=np.int64)
    else:
        n_out = int(round(spec.outlier_frac * spec.K))
        ch = np.sort(rng.choice(spec.K, size=n_out, replace=False))
    if spec.outlier_scale is not None:
        X[:, ch] *= np.float32(spec.outlier_scale)
    else:
        scale = rng.uniform(spec.outlier_lo, spec.outlier_hi, size=ch.shape[0]).astype(np.float32)
        X[:, ch] *= scale[None, :]
    return f32_to_bf16_bits(X)


def make_layer(spec: LayerSpec, M: int | None = None, seed_offset: int = 0) -> dict:
    """All bf16 inputs of one layer, drawn in a fixed order from one seed."""
    rng = np.random.default_rng(spec.seed + seed_offset)
    X = make_activations(spec, rng, M)
    W = f32_to_bf16_bits(rng.standard_normal((spec.N, spec.K), dtype=np.float32) * np.float32(spec.w_std))
    out = dict(X=X, W=W, L1=None, L2=None, bias=None)
    if spec.rank > 0:
        out["L1"] = f32_to_bf16_bits(rng.standard_normal((spec.K, spec.rank), dtype=np.float32) * np.float32(spec.lr_std))
        out["L2"] = f32_to_bf16_bits(rng.standard_normal((spec.rank, spec.N), dtype=np.float32) * np.float32(spec.lr_std))
    if spec.bias:
        out["bias"] = f32_to_bf16_bits(rng.standard_normal((spec.N,), dtype=np.float32) * np.float32(spec.b_std))
    return out


def random_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))
