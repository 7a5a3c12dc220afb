"""Number formats used by the SVDQuant W4A4 layer (oracle; test infrastructure).

The pages name the formats only: "nvfp4" with group_size 16 for svdq_w4a4
and "int4" (Nunchaku 4-bit in Diffusers, "Native Ladefunktion" config block),
computed in "bfloat16" (compute_dtype, same block).  The value sets below are
those formats' definitions:

  * E2M1 (the NVFP4 element): sign, 2 exponent bits (bias 1), 1 mantissa bit;
    magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.
  * E4M3 (the NVFP4 block scale; finite-only variant): 4 exponent bits
    (bias 7), 3 mantissa bits, subnormals, largest finite 448, no infinity.
  * fp16 (the INT4 group scale), bf16 (activations, low-rank factors, output).

Rounding is round-to-nearest, ties to the even significand ("RNE") in every
format.  "satfinite" clamps a finite out-of-range result to the largest
finite magnitude, keeping the sign.

The rounding is done on exact fp64 arithmetic: a value x with frexp exponent
e (|x| in [2^(e-1), 2^e)) has ulp 2^(e-p) in a format with p significand
bits, so RNE(x) = rint(x * 2^(p-e)) * 2^(e-p); both scalings are exact and
numpy's rint rounds half to even.  Subnormals use the smallest normal
exponent for e.
"""
from __future__ import annotations

import numpy as np

# (significand bits incl. the implicit one, smallest frexp exponent of a normal)
_BF16 = (8, -125)
_FP16 = (11, -13)
_E4M3 = (4, -5)
_E2M1 = (2, 1)

E4M3_MAX = 448.0
E2M1_MAX = 6.0
FP16_MAX = 65504.0
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def _rne(x, p: int, emin: int) -> np.ndarray:
    x = np.asarray(x, dtype=np.float64)
    _, e = np.frexp(x)
    e = np.maximum(e, emin)
    scale = np.ldexp(1.0, p - e)
    return np.rint(x * scale) / scale


def f32(x) -> np.ndarray:
    """Round to IEEE binary32 (numpy's cast is RNE)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16_rn(x) -> np.ndarray:
    """Round (fp64 or fp32) values to bf16, RNE; returned as fp64 values."""
    return _rne(x, *_BF16)


def fp16_rn(x) -> np.ndarray:
    """Round to IEEE binary16, RNE, overflow to +-inf; returned as fp64."""
    r = _rne(x, *_FP16)
    return np.where(np.abs(r) > FP16_MAX, np.copysign(np.inf, r), r)


def e4m3_rn_satfinite(x) -> np.ndarray:
    """Round to E4M3 (RNE) and clamp finite overflow to +-448; fp64 values."""
    r = _rne(x, *_E4M3)
    return np.clip(r, -E4M3_MAX, E4M3_MAX)


def e2m1_rn_satfinite(x) -> np.ndarray:
    """Round to E2M1 (RNE) and clamp finite overflow to +-6; fp64 values.
    The sign of a result that rounds to zero is kept (-0.0)."""
    r = _rne(x, *_E2M1)
    return np.where(np.abs(r) > E2M1_MAX, np.copysign(E2M1_MAX, r), r)


def e4m3_encode(v) -> np.ndarray:
    """E4M3 byte of a non-negative value that is already on the E4M3 grid."""
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(v > E4M3_MAX):
        raise ValueError("e4m3_encode expects grid values in [0, 448]")
    out = np.zeros(v.shape, dtype=np.uint8)
    sub = (v > 0) & (v < 2.0 ** -6)
    out[sub] = np.rint(v[sub] / 2.0 ** -9).astype(np.uint8)
    nrm = v >= 2.0 ** -6
    _, f = np.frexp(v[nrm])
    e = f - 1
    man = np.rint((v[nrm] / np.ldexp(1.0, e) - 1.0) * 8.0).astype(np.int64)
    out[nrm] = (((e + 7) << 3) | man).astype(np.uint8)
    return out


def e4m3_decode(code) -> np.ndarray:
    """Value of an E4M3 byte (sign bit honoured; 0x7F/0xFF are NaN)."""
    c = np.asarray(code, dtype=np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    ex = (c >> 3) & 0xF
    man = c & 7
    val = np.where(ex == 0, man * 2.0 ** -9, (1.0 + man / 8.0) * np.ldexp(1.0, ex - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return s * val


def e2m1_encode(v) -> np.ndarray:
    """E2M1 nibble (bit 3 = sign) of a value already on the E2M1 grid."""
    v = np.asarray(v, dtype=np.float64)
    mag = np.abs(v)
    idx = np.searchsorted(E2M1_GRID, mag)
    if np.any(idx >= 8) or np.any(E2M1_GRID[np.minimum(idx, 7)] != mag):
        raise ValueError("e2m1_encode expects E2M1 grid values")
    sign = np.signbit(v).astype(np.uint8)
    return (idx.astype(np.uint8) | (sign << 3)).astype(np.uint8)


def e2m1_decode(nib) -> np.ndarray:
    n = np.asarray(nib, dtype=np.int64)
    mag = E2M1_GRID[n & 7]
    return np.where(n & 8, -mag, mag)


def int4_to_nibble(q) -> np.ndarray:
    """Two's-complement nibble of an integer in [-8, 7]."""
    q = np.asarray(q, dtype=np.int64)
    if np.any(q < -8) or np.any(q > 7):
        raise ValueError("int4 out of range")
    return (q & 0xF).astype(np.uint8)


def nibble_to_int4(n) -> np.ndarray:
    n = np.asarray(n, dtype=np.int64) & 0xF
    return np.where(n >= 8, n - 16, n)


def pack_nibbles(nib: np.ndarray) -> np.ndarray:
    """Pack nibbles along the last axis, two per byte, even index in the low
    nibble."""
    nib = np.asarray(nib, dtype=np.uint8)
    if nib.shape[-1] % 2:
        raise ValueError("odd length")
    return (nib[..., 0::2] & 0xF) | ((nib[..., 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out
