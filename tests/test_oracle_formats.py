"""Pins of the oracle's number formats against the formats' definitions,
brute force, and library conversions (no GPU)."""
import os

import numpy as np
import pytest
import torch

from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_pairs(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        a, b = line.split()
        rows.append((a, b))
    return rows


def test_bf16_exhaustive_fixed_points():
    bits = np.arange(1 << 16, dtype=np.uint32)
    vals = (bits << 16).view(np.float32)
    vals = vals[np.isfinite(vals)]
    r = F.bf16_rn(vals)
    assert np.array_equal(r.astype(np.float32).view(np.uint32), vals.view(np.uint32))


def test_bf16_matches_torch_on_fp32():
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 10,
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),  # bf16 subnormals
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 2 ** -133, 3 * 2 ** -134], np.float32),
    ])
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(F.bf16_rn(x).astype(np.float32), ref)


def test_bf16_single_rounding_from_fp64():
    # 1 + 2^-8 + 2^-40 lies just above the bf16 tie 1 + 2^-8; going through
    # fp32 first would land on the tie and round down to 1.0.
    x = np.array([1 + 2.0 ** -8 + 2.0 ** -40, 1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8])
    assert F.bf16_rn(x).tolist() == [1 + 2.0 ** -7, 1.0, 1 + 2.0 ** -6]


def test_fp16_matches_numpy_cast():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 100,
        (rng.standard_normal(50000) * 1e-5).astype(np.float32),  # fp16 subnormals
        np.array([65504, 65519.99, 65520, 1e6, -70000, 2 ** -24, 2 ** -25, 3 * 2 ** -26], np.float32),
    ])
    with np.errstate(over="ignore"):  # 1e6 and -70000 overflow to +-inf on purpose
        ref = x.astype(np.float16).astype(np.float64)
    got = F.fp16_rn(x)
    assert np.array_equal(got, ref)


def test_e4m3_golden_codes():
    for code, val in _read_pairs("e4m3_values.txt"):
        c = int(code, 16)
        assert F.e4m3_decode(c) == float(val)
        assert int(F.e4m3_encode(float(val))) == c


def test_e4m3_all_codes_round_trip():
    codes = np.array([c for c in range(0x7F)], dtype=np.uint8)
    vals = F.e4m3_decode(codes)
    assert np.all(np.diff(vals) > 0)  # monotone in the code
    assert np.array_equal(F.e4m3_encode(vals), codes)
    assert np.array_equal(F.e4m3_rn_satfinite(vals), vals)


def test_e4m3_rounding_brute_force():
    grid = F.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    rng = np.random.default_rng(2)
    v = np.concatenate([
        np.exp(rng.uniform(np.log(1e-4), np.log(600), 100000)),
        (grid[:-1] + grid[1:]) / 2,  # exact ties
        rng.uniform(0, 2 ** -6, 5000),
    ]).astype(np.float32).astype(np.float64)
    d = np.abs(v[:, None] - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among equidistant candidates take the even code (even mantissa LSB)
    idx = np.where(cand & (np.arange(0x7F)[None, :] % 2 == 0), np.arange(0x7F)[None, :], 10 ** 6).min(axis=1)
    single = cand.sum(axis=1) == 1
    idx = np.where(single, np.argmax(cand, axis=1), idx)
    ref = grid[idx]
    ref = np.where(v > 448, 448.0, ref)
    assert np.array_equal(F.e4m3_rn_satfinite(v), ref)


def test_e4m3_matches_torch_in_range():
    rng = np.random.default_rng(3)
    v = np.exp(rng.uniform(np.log(1e-4), np.log(448), 200000)).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).to(torch.float32).numpy().astype(np.float64)
    assert np.array_equal(F.e4m3_rn_satfinite(v.astype(np.float64)), ref)


def test_e2m1_golden_table_and_ties():
    rows = _read_pairs("e2m1_values.txt")
    table = rows[:16]
    for code, val in table:
        got = F.e2m1_decode(int(code))
        assert got == float(val) and np.signbit(got) == val.startswith("-")
        assert int(F.e2m1_encode(float(val))) == int(code)
    for inp, exp in rows[16:]:
        got = F.e2m1_rn_satfinite(float(inp))
        assert got == float(exp) and np.signbit(got) == exp.startswith("-"), (inp, got, exp)


def test_e2m1_rounding_brute_force():
    grid = F.E2M1_GRID
    rng = np.random.default_rng(4)
    mag = np.concatenate([rng.uniform(0, 7, 200000), (grid[:-1] + grid[1:]) / 2]).astype(np.float32).astype(np.float64)
    d = np.abs(mag[:, None] - grid[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    ar = np.arange(8)[None, :]
    idx = np.where(cand & (ar % 2 == 0), ar, 99).min(axis=1)
    idx = np.where(cand.sum(axis=1) == 1, np.argmax(cand, axis=1), idx)
    ref = np.where(mag > 6, 6.0, grid[idx])
    assert np.array_equal(F.e2m1_rn_satfinite(mag), ref)
    assert np.array_equal(F.e2m1_rn_satfinite(-mag), -ref)


def test_int4_nibbles_and_packing():
    q = np.arange(-8, 8)
    n = F.int4_to_nibble(q)
    assert n.tolist() == [8, 9, 10, 11, 12, 13, 14, 15, 0, 1, 2, 3, 4, 5, 6, 7]
    assert np.array_equal(F.nibble_to_int4(n), q)
    packed = F.pack_nibbles(np.array([[1, 2, 3, 4]], np.uint8))
    assert packed.tolist() == [[0x21, 0x43]]  # even index in the low nibble
    assert np.array_equal(F.unpack_nibbles(packed), [[1, 2, 3, 4]])
    with pytest.raises(ValueError):
        F.int4_to_nibble(8)
