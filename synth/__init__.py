"""Seeded synthetic inputs for the SVDQuant W4A4 linear layer.

This module is the only code shared by the CPU oracle and the CUDA path.  It
draws the raw layer inputs (activations X, dense weights W, bias b) with the
shapes and value distributions of the FLUX-shaped diffusion-transformer
linears that the Nunchaku pages discuss, and holds none of the method's
arithmetic: no smoothing, no factorisation, no quantisation.

Inputs are returned as numpy arrays on the host:
  * X    : (M, K) float32 whose values are exactly representable in bf16,
           plus the raw bf16 bit patterns (uint16) for upload;
  * W    : (N, K) float32 (PyTorch nn.Linear orientation, out x in);
  * bias : (N,) float32 whose values are bf16-representable, plus bits.

Every draw is keyed by (workload, seed), so both sides see the same bytes.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "LayerShape",
    "LayerInputs",
    "WORKLOADS",
    "make_layer",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
    "qkv_prologue_inputs",
    "svd_start_block",
]


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even) and return the
    16-bit patterns.  Used only to store generated inputs in bf16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    flat = a.reshape(-1)
    out = np.empty(flat.shape, np.uint16)
    step = 1 << 20  # blocks of a million values keep the temporaries in cache
    for i in range(0, flat.size, step):
        u = flat[i:i + step].view(np.uint32).astype(np.uint64)
        lsb = (u >> np.uint64(16)) & np.uint64(1)
        out[i:i + step] = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return out.reshape(a.shape)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    name: str
    M: int
    K: int
    N: int
    rank: int
    precision: str  # "nvfp4" or "int4"
    group_size: int
    x_dist: str  # see _draw_x
    w_dist: str  # "gauss" or "gauss+spike"


@dataclasses.dataclass
class LayerInputs:
    shape: LayerShape
    seed: int
    x_bits: np.ndarray  # (M, K) uint16 bf16 patterns
    x: np.ndarray  # (M, K) float32, bf16-exact
    w: np.ndarray  # (N, K) float32
    bias_bits: np.ndarray  # (N,) uint16
    bias: np.ndarray  # (N,) float32, bf16-exact


# The five workloads: the tiny case, the FLUX-shaped fused QKV projection, the
# FLUX-shaped MLP pair, the INT4 four-image batch, and one linear shape of the
# 57-block denoising stack (all four block shapes are listed under "stack").
WORKLOADS = {
    "tiny": LayerShape("tiny", 64, 256, 256, 16, "nvfp4", 16, "outlier4x50", "gauss"),
    "qkv": LayerShape("qkv", 4608, 3072, 9216, 32, "nvfp4", 16, "outlier1pct", "gauss+spike"),
    "mlp_up": LayerShape("mlp_up", 4608, 3072, 12288, 32, "nvfp4", 16, "outlier1pct", "gauss"),
    "mlp_down": LayerShape("mlp_down", 4608, 12288, 3072, 32, "nvfp4", 16, "gelu1.5", "gauss"),
    "int4": LayerShape("int4", 18432, 3072, 3072, 32, "int4", 64, "student3", "gauss"),
    "stack_qkv": LayerShape("stack_qkv", 4608, 3072, 9216, 32, "nvfp4", 16, "outlier4x50", "gauss"),
    "stack_out": LayerShape("stack_out", 4608, 3072, 3072, 32, "nvfp4", 16, "outlier4x50", "gauss"),
    "stack_up": LayerShape("stack_up", 4608, 3072, 12288, 32, "nvfp4", 16, "outlier4x50", "gauss"),
    "stack_down": LayerShape("stack_down", 4608, 12288, 3072, 32, "nvfp4", 16, "outlier4x50", "gauss"),
    # the awq_w4a16 family: a FLUX double block's adaLN modulation (conditioning
    # vector after SiLU, 3072 -> 6 x 3072), one row per image
    "awq": LayerShape("awq", 1, 3072, 18432, 0, "awq", 64, "silu", "gauss"),
}

STACK_BLOCKS = 57
STACK_LAYERS = ("stack_qkv", "stack_out", "stack_up", "stack_down")


def _gelu_tanh(v: np.ndarray) -> np.ndarray:
    c = math.sqrt(2.0 / math.pi)
    return 0.5 * v * (1.0 + np.tanh(c * (v + 0.044715 * v ** 3)))


def _draw_x(rng: np.random.Generator, M: int, K: int, dist: str) -> np.ndarray:
    if dist == "outlier4x50":
        x = rng.standard_normal((M, K), dtype=np.float32)
        ch = rng.choice(K, size=min(4, K), replace=False)
        x[:, ch] *= np.float32(50.0)
        return x
    if dist == "outlier1pct":
        x = rng.standard_normal((M, K), dtype=np.float32)
        n_out = max(1, int(round(0.01 * K)))
        ch = rng.choice(K, size=n_out, replace=False)
        f = np.exp(rng.uniform(math.log(20.0), math.log(100.0), size=n_out)).astype(np.float32)
        x[:, ch] *= f[None, :]
        return x
    if dist == "gelu1.5":
        v = rng.standard_normal((M, K), dtype=np.float32) * np.float32(1.5)
        return _gelu_tanh(v.astype(np.float64)).astype(np.float32)
    if dist == "silu":  # SiLU of N(0, 1): the conditioning input of a modulation projection
        v = rng.standard_normal((M, K)).astype(np.float64)
        return (v / (1.0 + np.exp(-v))).astype(np.float32)
    if dist == "student3":
        return (0.5 * rng.standard_t(3.0, size=(M, K))).astype(np.float32)
    raise ValueError(dist)


def _draw_w(rng: np.random.Generator, N: int, K: int, dist: str) -> np.ndarray:
    w = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    if dist == "gauss":
        return w
    if dist == "gauss+spike":
        # rank-4 spike, each component of norm 10x the Gaussian part's
        # spectral norm (~0.02 * (sqrt(K) + sqrt(N))).
        sigma = 10.0 * 0.02 * (math.sqrt(K) + math.sqrt(N))
        spike = np.zeros((N, K), dtype=np.float64)
        for _ in range(4):
            u = rng.standard_normal(N)
            v = rng.standard_normal(K)
            u /= np.linalg.norm(u)
            v /= np.linalg.norm(v)
            spike += sigma * np.outer(u, v)
        return (w.astype(np.float64) + spike).astype(np.float32)
    raise ValueError(dist)


def make_layer(shape: LayerShape | str, seed: int, **overrides) -> LayerInputs:
    """Draw one layer's inputs.  Keyword overrides (M, K, N, rank, ...) give a
    reduced case with the same distributions; the draw is made for the
    overridden sizes, it is not a slice of the full-size draw."""
    if isinstance(shape, str):
        shape = WORKLOADS[shape]
    if overrides:
        shape = dataclasses.replace(shape, **overrides)
    rng = np.random.Generator(np.random.PCG64(seed))
    w = _draw_w(rng, shape.N, shape.K, shape.w_dist)
    bias = rng.standard_normal(shape.N, dtype=np.float32) * np.float32(0.01)
    x = _draw_x(rng, shape.M, shape.K, shape.x_dist)
    x_bits = bf16_bits_from_f32(x)
    b_bits = bf16_bits_from_f32(bias)
    return LayerInputs(shape, seed, x_bits, f32_from_bf16_bits(x_bits), w, b_bits, f32_from_bf16_bits(b_bits))


def stack_seed(block: int, layer: int) -> int:
    """Per-linear seed of the 57-block stack (4 linears per block)."""
    return 5000 + 4 * block + layer


def qkv_prologue_inputs(M: int, head_dim: int, seed: int):
    """Inputs of the fused QKV attention prologue: per-dimension RMS-norm
    weights for Q and K (fp32, uniform in [0.5, 1.5], like trained
    QK-norm scales around 1) and per-token rotary tables (fp32 cosines and
    sines of angles drawn uniformly in [-pi, pi), M x head_dim/2), drawn
    from (seed, M, head_dim)."""
    rng = np.random.default_rng([seed, M, head_dim, 7])
    norm_q = rng.uniform(0.5, 1.5, head_dim).astype(np.float32)
    norm_k = rng.uniform(0.5, 1.5, head_dim).astype(np.float32)
    ang = rng.uniform(-math.pi, math.pi, (M, head_dim // 2))
    return norm_q, norm_k, np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def awq_alpha(K: int, seed: int) -> np.ndarray:
    """An activation-aware per-input-channel scale for the awq_w4a16 layer:
    positive fp32 factors exp(U(-0.5, 0.5)) (a calibration would put them
    near 1), drawn from (seed, K)."""
    rng = np.random.default_rng([seed, K, 11])
    return np.exp(rng.uniform(-0.5, 0.5, K)).astype(np.float32)


def svd_start_block(n: int, ell: int, seed: int) -> np.ndarray:
    """The Gaussian start block of the randomized subspace iteration that
    factorises the smoothed weight (n x ell fp32, n = output features),
    drawn from (seed, n, ell)."""
    rng = np.random.default_rng([seed, n, ell, 13])
    return rng.standard_normal((n, ell)).astype(np.float32)
