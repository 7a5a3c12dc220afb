"""Pins of the oracle's NVFP4 / INT4 group quantisers (no GPU): grid-exact
round trips, brute-force element rounding, error bounds, special cases."""
import os

import numpy as np

from oracle import formats as F
from oracle import quant as Q

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_group_sizes_match_config_block():
    kv = dict(l.split() for l in open(os.path.join(GOLDEN, "config_block.txt")) if l.strip() and not l.startswith("#"))
    assert int(kv["svdq_w4a4.group_size"]) == Q.NVFP4_GROUP
    assert int(kv["awq_w4a16.group_size"]) == Q.INT4_GROUP
    assert kv["svdq_w4a4.precision"] == "nvfp4" and kv["awq_w4a16.precision"] == "int4"


def test_tensor_scale_rule():
    assert Q.nvfp4_tensor_scale(0.0) == np.float32(1.0)
    assert Q.nvfp4_tensor_scale(2688.0) == np.float32(1.0)
    assert Q.nvfp4_tensor_scale(5376.0) == np.float32(2.0)


def _grid_exact_groups(rng, n_groups):
    """Groups x = e * s * g whose largest |e| is 6, with s on the E4M3 grid and g
    a power of two: the quantiser must return exactly (e, s)."""
    grid = F.E2M1_GRID
    e = rng.choice(np.concatenate([grid, -grid]), size=(n_groups, 16))
    e[:, 0] = np.where(rng.random(n_groups) < 0.5, 6.0, -6.0)
    s_codes = rng.integers(1, 0x7F, size=n_groups).astype(np.uint8)
    s = F.e4m3_decode(s_codes)
    g = np.float32(2.0 ** -7)
    x = (e * s[:, None] * float(g)).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), e * s[:, None] * float(g))  # exact in fp32
    return x, e, s_codes, g


def test_nvfp4_grid_exact_round_trip():
    rng = np.random.default_rng(10)
    x, e, s_codes, g = _grid_exact_groups(rng, 4000)
    codes, sq = Q.nvfp4_quantize(x.reshape(-1, 16 * 8), g)
    codes = codes.reshape(-1, 16)
    sq = sq.reshape(-1)
    assert np.array_equal(sq, s_codes)
    dec = F.e2m1_decode(codes)
    assert np.array_equal(np.abs(dec), np.abs(e))
    assert np.array_equal(Q.nvfp4_dequantize(codes.reshape(-1, 128), sq.reshape(-1, 8), g).reshape(-1, 16), x)


def test_nvfp4_element_choice_is_nearest_grid_point():
    rng = np.random.default_rng(11)
    x = (rng.standard_normal((64, 256)) * np.exp(rng.uniform(-3, 3, (64, 1)))).astype(np.float32)
    g = Q.nvfp4_tensor_scale(np.abs(x).max())
    codes, sq = Q.nvfp4_quantize(x, g)
    s = F.e4m3_decode(sq).astype(np.float32)
    rcp = (np.float32(1) / (s * g)).astype(np.float32)
    v = (x.reshape(64, 16, 16) * rcp[:, :, None]).astype(np.float64)
    cand = np.concatenate([F.E2M1_GRID, -F.E2M1_GRID])
    dec = F.e2m1_decode(codes).reshape(v.shape)
    err = np.abs(dec - v)
    best = np.min(np.abs(v[..., None] - cand), axis=-1)
    best = np.where(np.abs(v) > 6, np.abs(v) - 6, best)
    assert np.array_equal(err, best)


def test_nvfp4_error_bound_and_scale_accuracy():
    rng = np.random.default_rng(12)
    x = (rng.standard_t(3, (256, 512))).astype(np.float32)
    g = Q.nvfp4_tensor_scale(np.abs(x).max())
    codes, sq = Q.nvfp4_quantize(x, g)
    deq = Q.nvfp4_dequantize(codes, sq, g)
    s = np.repeat(F.e4m3_decode(sq), 16, axis=1)
    step = s * float(g)
    err = np.abs(deq - x)
    # half of the widest E2M1 gap (4 -> 6) times the group's scale
    assert np.all(err <= 1.0 * step * (1 + 1e-6))
    small = np.abs(x) < 2 * step * 0.999
    assert np.all(err[small] <= 0.25 * step[small] * (1 + 1e-6))
    amax = np.abs(x.reshape(256, -1, 16)).max(axis=2)
    ideal = amax / 6 / float(g)
    sv = F.e4m3_decode(sq)
    nrm = ideal >= 2 ** -6
    assert np.all(np.abs(sv[nrm] - ideal[nrm]) <= ideal[nrm] * 2 ** -4 * (1 + 1e-6))


def test_nvfp4_zero_and_tiny_groups():
    x = np.zeros((2, 32), np.float32)
    x[1, 16:] = 1e-9  # amax/6/g far below the smallest E4M3 subnormal
    codes, sq = Q.nvfp4_quantize(x, np.float32(1.0))
    assert np.all(codes == 0) and np.all(sq == 0)


def test_nvfp4_negative_zero_reading():
    # a small negative value in a group with a nonzero scale rounds to -0,
    # stored as the nibble 0x8 (sign kept)
    x = np.zeros((1, 16), np.float32)
    x[0, 0] = 6.0
    x[0, 1] = -0.2
    codes, sq = Q.nvfp4_quantize(x, np.float32(1.0))
    assert F.e4m3_decode(sq[0, 0]) == 1.0
    assert codes[0, 0] == 7 and codes[0, 1] == 8 and codes[0, 2] == 0


def test_int4_grid_exact_round_trip():
    rng = np.random.default_rng(13)
    n = 3000
    q = rng.integers(-7, 8, size=(n, 64))
    q[:, 0] = np.where(rng.random(n) < 0.5, 7, -7)
    s = F.fp16_rn(np.exp(rng.uniform(np.log(1e-3), np.log(100), n)))
    x = (q * s[:, None]).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), q * s[:, None])
    qq, sh = Q.int4_quantize(x.reshape(-1, 64 * 4))
    assert np.array_equal(qq.reshape(-1, 64), q)
    assert np.array_equal(sh.reshape(-1).astype(np.float64), s)


def test_int4_brute_force_rounding():
    rng = np.random.default_rng(14)
    x = (rng.standard_normal((128, 256)) * 3).astype(np.float32)
    q, sh = Q.int4_quantize(x)
    s32 = sh.astype(np.float32)
    rcp = np.float32(1) / s32
    v = (x.reshape(128, 4, 64) * rcp[:, :, None]).astype(np.float64)
    ints = np.arange(-8, 8)
    d = np.abs(v[..., None] - ints)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    even = np.where(cand & (ints % 2 == 0), ints, 99).min(axis=-1)
    ref = np.where(cand.sum(-1) == 1, ints[np.argmax(cand, axis=-1)], even)
    assert np.array_equal(q.reshape(v.shape), ref)
    amax = np.abs(x.reshape(128, 4, 64)).max(axis=2)
    assert np.all(np.abs(sh.astype(np.float64) - amax / 7) <= amax / 7 * 2 ** -11 * (1 + 1e-6))


def test_int4_zero_group():
    q, sh = Q.int4_quantize(np.zeros((1, 64), np.float32))
    assert np.all(q == 0) and sh[0, 0] == 0
