"""The oracle's group quantisers against the same scale and rounding rules
carried out in exact rational arithmetic.

The oracle writes each rule as a chain of numpy fp32 operations (NVFP4:
s = E4M3(RN32(RN32(amax / 6) / g)), v = RN32(x * RN32(1 / RN32(s * g))),
code = E2M1(v); INT4: s_h = fp16(RN32(amax / 7)), q = rint(RN32(x *
RN32(1 / s_h))) clamped to [-8, 7]).  Here every rounding is done from its
IEEE definition on Fractions: round to nearest, ties to even, for binary32
(24-bit significand, subnormals down to 2^-149) and binary16 (11 bits,
subnormals down to 2^-24), and nearest-value search over the E4M3 and E2M1
grids (ties to the even code, saturating at the largest finite value).
Nothing below calls numpy's float32 arithmetic or the oracle's format
helpers, so a slip in the oracle's chain (an operation evaluated in fp64,
a step out of order, a wrong tie rule, a scale that is not saturated) shows
up as a differing code or scale byte.  Inputs span about 2^-30 .. 2^30 in
magnitude, so the E4M3 scales reach their subnormal range and zero.
"""
import math
import os
from fractions import Fraction

import numpy as np

from oracle import quant as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rn_binary(a: Fraction, mant_bits: int, emin: int, emax: int) -> Fraction | float:
    """Round a >= 0 to the nearest value of a binary format with `mant_bits`
    significand bits (hidden bit included), normal exponents emin .. emax;
    ties to even.  Returns math.inf on overflow."""
    if a == 0:
        return Fraction(0)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1  # now 2^e <= a < 2^(e + 1)
    ulp = Fraction(2) ** (max(e, emin) - (mant_bits - 1))
    m = a / ulp
    n = m.numerator // m.denominator
    r = m - n
    if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
        n += 1
    v = n * ulp
    if v >= Fraction(2) ** (emax + 1):
        return math.inf
    return v


def rn32(q: Fraction):
    if q < 0:
        v = rn32(-q)
        return -v
    return _rn_binary(q, 24, -126, 127)


def rn16(q: Fraction):
    return _rn_binary(q, 11, -14, 15)


def _e4m3_values():
    """(code, value) of every finite non-negative E4M3 code, from the format:
    4 exponent bits with bias 7, 3 mantissa bits, subnormals, 0x7F = NaN."""
    out = []
    for c in range(0x7F):
        e, m = c >> 3, c & 7
        v = Fraction(m, 8) * Fraction(2) ** -6 if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        out.append((c, v))
    return out


E4M3 = _e4m3_values()
E2M1 = [(c, Fraction(v)) for c, v in enumerate(["0", "0.5", "1", "1.5", "2", "3", "4", "6"])]


def _nearest_code(a: Fraction, table) -> int:
    """Nearest grid value to a >= 0 (ties to the even code), saturating."""
    if a >= table[-1][1]:
        return table[-1][0]
    best = min(table, key=lambda cv: (abs(cv[1] - a), cv[0] % 2))
    return best[0]


def test_e4m3_enumeration_matches_golden_table():
    vals = dict(E4M3)
    n = 0
    for line in open(os.path.join(GOLDEN, "e4m3_values.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        code, val = line.split()
        c = int(code, 16)
        if c < 0x7F:
            assert vals[c] == Fraction(val)
            n += 1
    assert n >= 8 and vals[0x7E] == 448


def _nvfp4_group_exact(x: np.ndarray, g: np.float32):
    """Codes and scale byte of one 16-group by exact arithmetic."""
    xs = [Fraction(float(v)) for v in x]
    G = Fraction(float(g))
    amax = max(abs(v) for v in xs)
    s_f = rn32(rn32(amax / 6) / G)
    s_code = _nearest_code(s_f, E4M3)
    s = dict(E4M3)[s_code]
    if s == 0:
        return [0] * 16, s_code
    rcp = rn32(1 / rn32(s * G))
    codes = []
    for xf, xv in zip(x, xs):
        v = rn32(xv * rcp)
        mag = _nearest_code(abs(v), E2M1)
        neg = xf < 0 or (xf == 0 and math.copysign(1.0, float(xf)) < 0)
        codes.append(mag | (8 if neg else 0))
    return codes, s_code


def _f32(q: Fraction) -> np.float32:
    v = rn32(q)
    return np.float32(float(v) if v != math.inf else np.inf)


def _nvfp4_boundary_groups(g: np.float32, rng) -> np.ndarray:
    """Groups whose values sit within a few fp32 ulps of a rounding boundary.

    - Scale boundaries: the group maximum puts amax / (6 g) next to the
      midpoint of two neighbouring E4M3 values (normal and subnormal).
    - Element boundaries: with the maximum fixed so that the scale is an
      exact E4M3 value s, the other entries put x / (s g) next to the
      midpoints of the E2M1 grid.  g = 0.1 makes s g and 1 / (s g)
      inexact, so the order and precision of the roundings decide the side.
    """
    G = Fraction(float(g))
    out = []
    vals = [v for _, v in E4M3]
    for i in (3, 10, 30, 56, 70, 90, 110):  # subnormal and normal neighbours
        t = (vals[i] + vals[i + 1]) / 2
        for k in range(-3, 4):
            amax = _f32(6 * t * G * (1 + Fraction(k, 1 << 24)))
            grp = np.concatenate([[amax], (amax * rng.uniform(-1, 1, 15)).astype(np.float32)])
            out.append(grp.astype(np.float32))
    # a scale past the largest E4M3 value (448): saturated, and the codes of
    # the larger entries saturate at 6 in turn
    amax = _f32(6 * 500 * G)
    out.append(np.concatenate([[amax], (amax * rng.uniform(-1, 1, 15)).astype(np.float32)]).astype(np.float32))
    mids = [Fraction(m) for m in ("0.25", "0.75", "1.25", "1.75", "2.5", "3.5", "5")]
    for s in (Fraction(3, 2), Fraction(5, 4), Fraction(13, 16), Fraction(7, 2)):
        amax = _f32(6 * s * G)  # its scale rounds back to s (checked below through the exact chain)
        for k in range(-2, 3):
            row = [amax]
            for j in range(15):
                m = mids[j % len(mids)]
                sign = -1 if j % 2 else 1
                row.append(_f32(sign * m * s * G * (1 + Fraction(k, 1 << 23))))
            out.append(np.array(row, np.float32))
    return np.stack(out)


def test_nvfp4_chain_matches_exact_arithmetic():
    rng = np.random.default_rng(20)
    groups = 160
    # each group its own magnitude, 2^-30 .. 2^30 around the tensor's
    mag = np.exp2(rng.uniform(-30, 30, (groups, 1)))
    x = (rng.standard_normal((groups, 16)) * mag).astype(np.float32)
    x[3, :] = 0.0  # an all-zero group
    x[5, 7] = -0.0
    x[9, :] = np.float32(2.0 ** -40) * np.sign(rng.standard_normal(16)).astype(np.float32)  # scale rounds to 0
    g = Q.nvfp4_tensor_scale(np.abs(x).max())
    codes, sq = Q.nvfp4_quantize(x.reshape(1, -1), g)
    codes = codes.reshape(groups, 16)
    sq = sq.reshape(groups)
    zero_scales = 0
    for b in range(groups):
        ec, es = _nvfp4_group_exact(x[b], g)
        assert int(sq[b]) == es, (b, int(sq[b]), es)
        assert codes[b].tolist() == ec, (b, codes[b].tolist(), ec)
        zero_scales += es == 0
    assert zero_scales >= 2  # the zero group and the one below the smallest scale


def test_nvfp4_chain_at_rounding_boundaries():
    rng = np.random.default_rng(22)
    g = np.float32(0.1)
    x = _nvfp4_boundary_groups(g, rng)
    codes, sq = Q.nvfp4_quantize(x.reshape(1, -1), g)
    codes = codes.reshape(len(x), 16)
    sq = sq.reshape(len(x))
    saturated = 0
    for b in range(len(x)):
        ec, es = _nvfp4_group_exact(x[b], g)
        assert int(sq[b]) == es, (b, int(sq[b]), es)
        assert codes[b].tolist() == ec, (b, codes[b].tolist(), ec)
        saturated += es == 0x7E
    assert saturated == 1


def _int4_group_exact(x: np.ndarray):
    xs = [Fraction(float(v)) for v in x]
    amax = max(abs(v) for v in xs)
    s_h = rn16(rn32(amax / 7))
    assert s_h != math.inf
    if s_h == 0:
        return [0] * 64, s_h
    rcp = rn32(1 / s_h)
    q = []
    for xv in xs:
        v = rn32(xv * rcp)
        n = math.floor(v)
        r = v - n
        if r > Fraction(1, 2) or (r == Fraction(1, 2) and n % 2 == 1):
            n += 1
        q.append(max(-8, min(7, n)))
    return q, s_h


def test_int4_chain_matches_exact_arithmetic():
    rng = np.random.default_rng(21)
    groups = 96
    mag = np.exp2(rng.uniform(-24, 15, (groups, 1)))  # up to ~3e4: fp16 scales stay finite
    x = (rng.standard_normal((groups, 64)) * mag).astype(np.float32)
    x[2, :] = 0.0
    x[4, :] = np.float32(2.0 ** -30)  # below half the smallest fp16 subnormal times 7: s_h = 0
    # scale 2^j exactly (amax = 7 * 2^j), entries (n + 1/2) 2^j: exact ties of rint
    for r, j in ((6, 0), (7, -3), (8, 5)):
        n = rng.integers(-7, 7, 64)  # |n + 1/2| <= 6.5 < 7: the first entry stays the maximum
        x[r, :] = ((n + 0.5) * 2.0 ** j).astype(np.float32)
        x[r, 0] = np.float32(7 * 2.0 ** j)
    # scale fp16(1.1): entries a few ulps either side of x * rcp = n + 1/2
    s_h = rn16(rn32(Fraction(77, 10) / 7))
    for r in (10, 11, 12, 13, 14):
        k = r - 12
        n = rng.integers(-7, 7, 64)  # |n + 1/2| s_h <= 7.15 < 7.7
        x[r, :] = [_f32((int(v) + Fraction(1, 2)) * s_h * (1 + Fraction(k, 1 << 24))) for v in n]
        x[r, 0] = np.float32(7.7)
    q, s_h = Q.int4_quantize(x.reshape(1, -1))
    q = q.reshape(groups, 64)
    s_h = s_h.reshape(groups)
    for b in range(groups):
        eq, es = _int4_group_exact(x[b])
        assert Fraction(float(s_h[b])) == es, (b, float(s_h[b]), es)
        assert q[b].tolist() == eq, (b, q[b].tolist(), eq)
