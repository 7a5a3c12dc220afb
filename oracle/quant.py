"""Group quantisers of the SVDQuant W4A4 layer (oracle; test infrastructure).

The pages state that both the weights' residual and the live activations are
quantised to 4 bits (Nunchaku 4-bit in Diffusers, "Nunchaku und SVDQuant";
ai2day "Was ist Nunchaku Lite"), in NVFP4 with a group of 16 or in INT4
("Native Ladefunktion" config block, "Hardware-Unterstuetzung").  They give
no scale rule and no rounding mode; the rules below are readings (the
plainest ones the pages support), written as a fixed sequence of IEEE fp32
operations so that a GPU can reproduce them bit for bit:

NVFP4, one group b of 16 values x (fp32) with a per-tensor fp32 scale g:
    amax_b = max |x|
    s_f    = RN32( RN32(amax_b / 6) / g )
    s_q    = E4M3_RNE_satfinite(s_f)            (the stored scale byte)
    s      = value(s_q)
    if s == 0: every code is +0
    else:      rcp = RN32(1 / RN32(s * g)); v = RN32(x * rcp)
               code = E2M1_RNE_satfinite(v)     (sign kept, -0 -> 0x8)
    dequantised value = e2m1(code) * s * g

INT4, one group of 64 values x (fp32):
    s_h = fp16_RN( RN32(amax / 7) )             (the stored fp16 scale)
    if s_h == 0: every code is 0
    else:       rcp = RN32(1 / float(s_h)); q = clamp(rint(RN32(x * rcp)), -8, 7)
    dequantised value = q * s_h

Tensor scale of an NVFP4 tensor: g = RN32(amax / 2688) with 2688 = 6 * 448
(the largest E2M1 magnitude times the largest E4M3 scale); g = 1 when amax
is 0.
"""
from __future__ import annotations

import numpy as np

from . import formats as F

NVFP4_GROUP = 16
INT4_GROUP = 64


def nvfp4_tensor_scale(amax) -> np.float32:
    amax = np.float32(amax)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax / np.float32(2688.0))


# Rows are independent, so the quantisers work through them in blocks of
# this many rows (keeps the temporaries small; the arithmetic per element is
# the same as on the whole matrix at once).
_ROW_BLOCK = 256


def _by_row_blocks(fn, x: np.ndarray):
    R = x.shape[0]
    if R <= _ROW_BLOCK:
        return fn(x)
    parts = [fn(x[i:i + _ROW_BLOCK]) for i in range(0, R, _ROW_BLOCK)]
    return tuple(np.concatenate([p[j] for p in parts], axis=0) for j in range(len(parts[0])))


def nvfp4_quantize(x: np.ndarray, g) -> tuple[np.ndarray, np.ndarray]:
    """Quantise rows of fp32 values, groups of 16 along the last axis.

    Returns (codes, scale_bytes): codes are E2M1 nibbles (uint8, one per
    element, bit 3 = sign), scale_bytes are E4M3 bytes, one per group.
    """
    x = np.asarray(x, dtype=np.float32)
    g = np.float32(g)
    if x.shape[1] % NVFP4_GROUP:
        raise ValueError("K must be a multiple of 16")
    return _by_row_blocks(lambda xb: _nvfp4_rows(xb, g), x)


def _nvfp4_rows(x: np.ndarray, g: np.float32) -> tuple[np.ndarray, np.ndarray]:
    R, K = x.shape
    xg = x.reshape(R, K // NVFP4_GROUP, NVFP4_GROUP)
    amax = np.max(np.abs(xg), axis=2)  # fp32, exact
    s_f = (amax / np.float32(6.0)) / g  # two fp32 divisions, each RN
    s_q = F.e4m3_encode(F.e4m3_rn_satfinite(s_f.astype(np.float64)))
    s = F.e4m3_decode(s_q).astype(np.float32)  # exact
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        rcp = np.float32(1.0) / (s * g)  # RN32(1 / RN32(s*g))
        v = xg * rcp[:, :, None]  # RN32
    codes = F.e2m1_encode(F.e2m1_rn_satfinite(np.where(s[:, :, None] == 0, 0.0, v).astype(np.float64)))
    codes = np.where(s[:, :, None] == 0, np.uint8(0), codes)
    return codes.reshape(R, K).astype(np.uint8), s_q.astype(np.uint8)


def nvfp4_dequantize(codes: np.ndarray, scale_bytes: np.ndarray, g) -> np.ndarray:
    """fp64 values e2m1(code) * s * g (exact products)."""
    R, K = codes.shape
    out = np.empty((R, K), np.float64)
    for i in range(0, R, _ROW_BLOCK):
        e = F.e2m1_decode(codes[i:i + _ROW_BLOCK]).reshape(-1, K // NVFP4_GROUP, NVFP4_GROUP)
        s = F.e4m3_decode(scale_bytes[i:i + _ROW_BLOCK])
        out[i:i + _ROW_BLOCK] = (e * s[:, :, None]).reshape(-1, K) * float(np.float32(g))
    return out


def int4_quantize(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Quantise rows of fp32 values, groups of 64 along the last axis.

    Returns (q, s_h): q int8 in [-8, 7] (one per element), s_h float16 (one
    per group).
    """
    x = np.asarray(x, dtype=np.float32)
    if x.shape[1] % INT4_GROUP:
        raise ValueError("K must be a multiple of 64")
    return _by_row_blocks(_int4_rows, x)


def _int4_rows(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    R, K = x.shape
    xg = x.reshape(R, K // INT4_GROUP, INT4_GROUP)
    amax = np.max(np.abs(xg), axis=2)
    s_h = F.fp16_rn((amax / np.float32(7.0)).astype(np.float64))  # fp64 values on the fp16 grid
    s32 = s_h.astype(np.float32)
    with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
        rcp = np.float32(1.0) / s32
        v = xg * rcp[:, :, None]
    q = np.clip(np.rint(np.where(s32[:, :, None] == 0, 0.0, v)), -8, 7).astype(np.int8)
    return q.reshape(R, K), s_h.astype(np.float16)


def int4_dequantize(q: np.ndarray, s_h: np.ndarray) -> np.ndarray:
    R, K = q.shape
    v = q.astype(np.float64).reshape(R, K // INT4_GROUP, INT4_GROUP)
    return (v * s_h.astype(np.float64)[:, :, None]).reshape(R, K)
