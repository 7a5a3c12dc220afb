"""Pins of the oracle's fused-QKV attention prologue (no GPU): closed forms
and invariants of the RMS normalisation and of the rotary embedding, and a
tiny worked example computed by hand."""
import math

import numpy as np

from oracle import qkv as A


def test_rotary_identity_at_zero_angle():
    rng = np.random.default_rng(0)
    y = rng.normal(size=(3, 8))
    c = np.ones((3, 4))
    s = np.zeros((3, 4))
    assert np.array_equal(A.rotary_pairs(y, c, s, 8), y)


def test_rotary_of_basis_vectors():
    # e_{2i} -> (cos, sin) at (2i, 2i+1); e_{2i+1} -> (-sin, cos)
    th = np.array([[0.3, -1.1]])
    c, s = np.cos(th), np.sin(th)
    for i in range(2):
        e = np.zeros((1, 4))
        e[0, 2 * i] = 1.0
        out = A.rotary_pairs(e, c, s, 4)
        want = np.zeros((1, 4))
        want[0, 2 * i], want[0, 2 * i + 1] = c[0, i], s[0, i]
        assert np.array_equal(out, want)
        e = np.zeros((1, 4))
        e[0, 2 * i + 1] = 1.0
        out = A.rotary_pairs(e, c, s, 4)
        want = np.zeros((1, 4))
        want[0, 2 * i], want[0, 2 * i + 1] = -s[0, i], c[0, i]
        assert np.array_equal(out, want)


def test_rotary_keeps_pair_norms_and_composes():
    rng = np.random.default_rng(1)
    y = rng.normal(size=(5, 16))
    t1 = rng.uniform(-3, 3, size=(5, 8))
    t2 = rng.uniform(-3, 3, size=(5, 8))
    r1 = A.rotary_pairs(y, np.cos(t1), np.sin(t1), 16)
    n0 = y.reshape(5, 8, 2)
    n1 = r1.reshape(5, 8, 2)
    assert np.allclose((n0 ** 2).sum(-1), (n1 ** 2).sum(-1), rtol=1e-12, atol=0)
    r12 = A.rotary_pairs(r1, np.cos(t2), np.sin(t2), 16)
    direct = A.rotary_pairs(y, np.cos(t1 + t2), np.sin(t1 + t2), 16)
    assert np.allclose(r12, direct, rtol=0, atol=1e-12)
    back = A.rotary_pairs(r1, np.cos(-t1), np.sin(-t1), 16)
    assert np.allclose(back, y, rtol=0, atol=1e-12)


def test_rms_norm_unit_mean_square_scale_invariance_and_constant():
    rng = np.random.default_rng(2)
    y = rng.normal(size=(4, 32)) * rng.uniform(0.1, 10, size=(4, 1))
    out = A.rms_norm_heads(y, np.ones(16), 16, 0.0)
    ms = (out.reshape(4, 2, 16) ** 2).mean(-1)
    assert np.allclose(ms, 1.0, rtol=1e-12, atol=0)
    assert np.allclose(A.rms_norm_heads(7.5 * y, np.ones(16), 16, 0.0), out, rtol=1e-12, atol=0)
    # a constant head c: every value becomes w * c / sqrt(c^2 + eps)
    c, eps = -3.0, 0.25
    w = np.arange(1, 5, dtype=np.float64)
    got = A.rms_norm_heads(np.full((1, 4), c), w, 4, eps)
    assert np.allclose(got, w * c / math.sqrt(c * c + eps), rtol=1e-15, atol=0)


def test_prologue_worked_example_by_hand():
    # heads = 1, head_dim = 4: Y = [q | k | v]
    q = [1.0, 2.0, 3.0, 4.0]        # mean square 7.5
    k = [2.0, 0.0, 0.0, 0.0]        # mean square 1
    v = [5.0, -6.0, 7.0, -8.0]
    y = np.array([q + k + v])
    cos = np.array([[0.0, 1.0]])    # pair 0 turned by +90 degrees, pair 1 kept
    sin = np.array([[1.0, 0.0]])
    wq = np.ones(4)
    wk = np.array([0.5, 1.0, 1.0, 1.0])
    out = A.qkv_prologue(y, 1, 4, wq, wk, cos, sin, eps=0.0)
    r = 1.0 / math.sqrt(7.5)
    # q: (1, 2) -> (-2, 1) by the quarter turn; (3, 4) unchanged
    assert np.allclose(out[0, 0:4], [-2 * r, 1 * r, 3 * r, 4 * r], rtol=1e-15, atol=0)
    # k: normalised (2, 0, 0, 0) / 1 * wk = (1, 0, 0, 0); quarter turn -> (0, 1)
    assert np.allclose(out[0, 4:8], [0.0, 1.0, 0.0, 0.0], rtol=0, atol=1e-15)
    assert np.array_equal(out[0, 8:12], v)


def test_prologue_passes_v_and_matches_per_section_steps():
    rng = np.random.default_rng(3)
    heads, d, m = 2, 8, 5
    y = rng.normal(size=(m, 3 * heads * d))
    c, s = A.rope_tables(np.arange(m), d)
    wq, wk = rng.uniform(0.5, 2, d), rng.uniform(0.5, 2, d)
    out = A.qkv_prologue(y, heads, d, wq, wk, c, s, 1e-6)
    assert np.array_equal(out[:, 2 * heads * d:], y[:, 2 * heads * d:])
    # every output head of Q and K keeps the squared norm of the weighted,
    # normalised input: rotations keep it, up to cos^2 + sin^2 = 1 within
    # the fp32 rounding of the tables (relative 2^-23 each)
    for sec, w in ((0, wq), (1, wk)):
        blk = out[:, sec * heads * d:(sec + 1) * heads * d].reshape(m, heads, d)
        src = y[:, sec * heads * d:(sec + 1) * heads * d].reshape(m, heads, d)
        nrm = src / np.sqrt((src ** 2).mean(-1, keepdims=True) + 1e-6)
        assert np.allclose((blk ** 2).sum(-1), ((nrm * w) ** 2).sum(-1), rtol=4e-7, atol=0)


def test_rope_tables_angles():
    c, s = A.rope_tables(np.array([0, 1, 7]), 8, theta=10000.0)
    assert np.array_equal(c[0], np.ones(4, np.float32)) and np.array_equal(s[0], np.zeros(4, np.float32))
    assert c[1, 0] == np.float32(math.cos(1.0)) and s[2, 0] == np.float32(math.sin(7.0))
    assert s[1, 2] == np.float32(math.sin(10000.0 ** -0.5))
