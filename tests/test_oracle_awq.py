"""Pins of the oracle's awq_w4a16 layer (no GPU)."""
import numpy as np

from oracle import awq as A
from oracle import formats as F


def _grid_weights(rng, N, K):
    """Weights already on the INT4 grid: every 64-group holds a 7 (so
    amax = 7 s) times a power-of-two scale s, the rest integers in [-7, 7]
    times s (a -8 would raise amax to 8 s).  The quantiser must reproduce
    them exactly."""
    q = rng.integers(-7, 8, size=(N, K))
    q[:, ::64] = 7
    s = rng.choice([0.25, 0.5, 1.0, 2.0], size=(N, K // 64))
    return (q * np.repeat(s, 64, axis=1)).astype(np.float32), q, s


def test_lossless_on_grid_weights_equals_plain_product():
    rng = np.random.default_rng(0)
    N, K, M = 48, 192, 5
    w, q, s = _grid_weights(rng, N, K)
    x = F.bf16_rn(rng.normal(size=(M, K))).astype(np.float32)
    b = F.bf16_rn(rng.normal(size=N) * 0.01).astype(np.float32)
    prep = A.prepare(w, np.ones(K, np.float32), b)
    assert np.array_equal(prep.q, q)
    assert np.array_equal(prep.s.astype(np.float64), s)
    # a separate naive product: sum over k of x * w, plus b, in fp64
    ref = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            ref[m, n] = sum(float(x[m, k]) * float(w[n, k]) for k in range(K)) + float(b[n])
    assert np.allclose(A.forward(x, prep), ref, rtol=0, atol=1e-9)


def test_alpha_moves_between_activations_and_weights():
    """With power-of-two alpha both roundings are exact, so the quantised
    layer with alpha equals the one without it on alpha-scaled weights."""
    rng = np.random.default_rng(1)
    N, K, M = 32, 128, 4
    w = (rng.normal(size=(N, K)) * 0.02).astype(np.float32)
    x = F.bf16_rn(rng.normal(size=(M, K))).astype(np.float32)
    b = np.zeros(N, np.float32)
    alpha = rng.choice([0.5, 1.0, 2.0, 4.0], size=K).astype(np.float32)
    with_alpha = A.forward(x, A.prepare(w, alpha, b))
    moved = A.forward((x / alpha).astype(np.float32), A.prepare(w * alpha, np.ones(K, np.float32), b))
    assert np.array_equal(with_alpha, moved)


def test_quantisation_error_bound():
    """Per element the 4-bit weight error is at most half a step s/2, so
    |Y* - X W^T| <= sum_k |x_k| s_g(k) / 2 (alpha = 1)."""
    rng = np.random.default_rng(2)
    N, K, M = 40, 256, 6
    w = (rng.normal(size=(N, K)) * 0.02).astype(np.float32)
    x = F.bf16_rn(rng.normal(size=(M, K))).astype(np.float32)
    prep = A.prepare(w, np.ones(K, np.float32), np.zeros(N, np.float32))
    y = A.forward(x, prep)
    exact = x.astype(np.float64) @ w.astype(np.float64).T
    step = np.repeat(prep.s.astype(np.float64), 64, axis=1)  # N x K
    bound = np.abs(x).astype(np.float64) @ (step / 2).T * (1 + 1e-3)
    assert np.all(np.abs(y - exact) <= bound)
