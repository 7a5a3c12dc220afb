"""Pins of the oracle's method steps (no GPU): smoothing, truncated SVD,
residual, forward assembly, and the low-rank branch's quality invariant."""
import numpy as np
import pytest

import synth
from oracle import formats as F
from oracle import quant as Q
from oracle import svd as S
from oracle import svdq as V


def test_lambda_closed_form_and_zero_channels():
    x = np.zeros((3, 4), np.float32)
    w = np.zeros((2, 4), np.float32)
    x[1, 0], w[0, 0] = -8.0, 0.5  # sqrt(8 / 0.5) = 4
    x[2, 1], w[1, 1] = 2.0, 8.0  # sqrt(2 / 8) = 0.5
    x[0, 2] = 3.0  # W column all zero -> 1
    w[1, 3] = 1.0  # X column all zero -> 1
    assert V.smoothing_lambda(x, w).tolist() == [4.0, 0.5, 1.0, 1.0]


def test_smoothing_preserves_the_product():
    li = synth.make_layer("tiny", 7)
    lam = V.smoothing_lambda(li.x, li.w)
    xh = V.smooth_activation(li.x, V.inv_lambda(lam)).astype(np.float64)
    wt = V.smooth_weight(li.w, lam).astype(np.float64)
    ref = li.x.astype(np.float64) @ li.w.astype(np.float64).T
    got = xh @ wt.T
    # two fp32 roundings per term: relative 2^-23 of sum |x||w|
    bound = 2.0 ** -22 * (np.abs(li.x) @ np.abs(li.w).T)
    assert np.all(np.abs(got - ref) <= bound)
    # after smoothing the per-channel maxima of X_hat and W_til agree
    mx = np.abs(xh).max(0)
    mw = np.abs(wt).max(0)
    assert np.allclose(mx, mw, rtol=1e-5)


def test_svd_diagonal_and_rank_one():
    A = np.diag([5.0, 3.0, 2.0, 1.0])
    U, s, Vv = S.truncated_svd(A, 2)
    assert np.allclose(s, [5.0, 3.0])
    assert np.allclose(np.abs(U.T @ A @ Vv), np.diag([5.0, 3.0]))
    u = np.arange(1.0, 7.0)
    v = np.array([1.0, -2.0, 0.5])
    U, s, Vv = S.truncated_svd(np.outer(u, v), 1)
    assert np.isclose(s[0], np.linalg.norm(u) * np.linalg.norm(v))
    assert np.allclose(s[0] * U @ Vv.T, np.outer(u, v))


def test_svd_eckart_young_tail():
    rng = np.random.default_rng(5)
    A = rng.standard_normal((60, 40))
    sv = np.linalg.svd(A, compute_uv=False)
    for r in (0, 1, 5, 17):
        U, s, Vv = S.truncated_svd(A, r)
        err = np.linalg.norm(A - (U * s) @ Vv.T) ** 2
        assert np.isclose(err, np.sum(sv[r:] ** 2))


def test_subspace_iteration_recovers_known_spectrum():
    rng = np.random.default_rng(6)
    m, n, r = 1500, 1100, 32
    Uq, _ = np.linalg.qr(rng.standard_normal((m, 64)))
    Vq, _ = np.linalg.qr(rng.standard_normal((n, 64)))
    sig = np.concatenate([np.geomspace(100, 10, 32), np.geomspace(1, 0.5, 32)])
    A = (Uq * sig) @ Vq.T + 1e-3 * rng.standard_normal((m, n))
    assert min(m, n) > S.EXACT_MAX_DIM
    U, s, Vv = S.truncated_svd(A, r)
    assert np.allclose(s, sig[:r], rtol=1e-3)
    assert np.allclose(U.T @ U, np.eye(r), atol=1e-10)


def test_residual_chain_is_exact_when_W_is_the_lowrank_product():
    # lambda = 1 and W = (L1 L2)^T built exactly from short bf16 values:
    # R must be exactly 0, every weight code 0, g_w = 1, and the forward must
    # reduce to the pure low-rank product X L1^T L2^T + b.
    rng = np.random.default_rng(8)
    K, N, r, M = 64, 48, 4, 24
    L1 = (rng.integers(-16, 17, (r, K)) / 8.0).astype(np.float32)
    L2 = (rng.integers(-16, 17, (N, r)) / 16.0).astype(np.float32)
    W = (L2.astype(np.float64) @ L1.astype(np.float64)).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), L2.astype(np.float64) @ L1.astype(np.float64))
    lam = np.ones(K, np.float32)
    b = F.bf16_rn(rng.standard_normal(N) * 0.1).astype(np.float32)
    prep = V.prepare_weights(W, lam, L1, L2, b)
    assert np.all(prep.R == 0) and prep.g_w == 1.0 and np.all(prep.qw == 0) and np.all(prep.sw == 0)
    x = F.bf16_rn(rng.standard_normal((M, K))).astype(np.float32)
    gx = V.act_global_scale(x, prep.inv_lam)
    y = V.forward(x, prep, gx)
    ref = (x.astype(np.float64) @ L1.astype(np.float64).T) @ L2.astype(np.float64).T + b
    assert np.allclose(y, ref, rtol=0, atol=1e-12)


def _naive_quantized_gemm(x, w, b):
    """lambda = 1, rank 0: Y = dequant(Q(X)) dequant(Q(W))^T + b, written as
    plain loops over elements with per-element dequantisation."""
    M, K = x.shape
    N = w.shape[0]
    gx = Q.nvfp4_tensor_scale(np.abs(x).max())
    gw = Q.nvfp4_tensor_scale(np.abs(w).max())
    cx, sx = Q.nvfp4_quantize(x, gx)
    cw, sw = Q.nvfp4_quantize(w, gw)
    y = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                ex = F.e2m1_decode(cx[m, k]) * F.e4m3_decode(sx[m, k // 16]) * float(gx)
                ew = F.e2m1_decode(cw[n, k]) * F.e4m3_decode(sw[n, k // 16]) * float(gw)
                acc += ex * ew
            y[m, n] = acc + b[n]
    return y, gx


def test_lambda1_rank0_equals_plain_quantized_gemm():
    rng = np.random.default_rng(9)
    M, K, N = 5, 48, 7
    x = F.bf16_rn(rng.standard_normal((M, K))).astype(np.float32)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    b = F.bf16_rn(rng.standard_normal(N) * 0.01).astype(np.float32)
    prep = V.prepare_weights(w, np.ones(K, np.float32), np.zeros((0, K), np.float32), np.zeros((N, 0), np.float32), b)
    ref, gx = _naive_quantized_gemm(x, w, b)
    assert gx == V.act_global_scale(x, prep.inv_lam)
    y = V.forward(x, prep, gx)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_int4_forward_is_group_sum():
    rng = np.random.default_rng(15)
    M, K, N, r = 6, 128, 5, 2
    li = synth.make_layer("int4", 3, M=M, K=K, N=N, rank=r)
    lam = V.smoothing_lambda(li.x, li.w)
    L1, L2 = V.lowrank_factors(li.w, lam, r)
    prep = V.prepare_weights(li.w, lam, L1, L2, li.bias, "int4")
    a = V.quantize_activations(li.x, prep)
    y = V.forward_from_codes(a, prep)
    ref = np.zeros((M, N))
    for m in range(M):
        for n in range(N):
            for g in range(K // 64):
                sl = slice(64 * g, 64 * g + 64)
                ref[m, n] += float(a.sx[m, g]) * float(prep.sw[n, g]) * int(np.dot(a.qx[m, sl].astype(np.int64), prep.qw[n, sl].astype(np.int64)))
            ref[m, n] += float(np.dot(li.x[m].astype(np.float64), prep.L1s.astype(np.float64).T) @ prep.L2[n].astype(np.float64))
            ref[m, n] += li.bias[n]
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-9)


@pytest.mark.parametrize("precision", ["nvfp4", "int4"])
def test_error_falls_as_rank_grows(precision):
    # the low-rank branch absorbs the hard part of W: the quantised layer's
    # error against the dense layer is non-increasing in the rank
    if precision == "nvfp4":
        li = synth.make_layer("qkv", 21, M=256, K=512, N=768)
    else:
        li = synth.make_layer("int4", 21, M=256, K=512, N=768)
    dense = V.reference_dense(li.x, li.w, li.bias)
    lam = V.smoothing_lambda(li.x, li.w)
    errs = []
    for r in (0, 4, 8, 16, 32):
        L1, L2 = V.lowrank_factors(li.w, lam, r)
        prep = V.prepare_weights(li.w, lam, L1, L2, li.bias, precision)
        gx = V.act_global_scale(li.x, prep.inv_lam)
        y = V.forward(li.x, prep, gx)
        errs.append(np.linalg.norm(y - dense) / np.linalg.norm(dense))
    for a, b in zip(errs, errs[1:]):
        assert b <= a * 1.01, errs
    # with a rank-4 spike in W the branch must take most of the error away;
    # with a purely Gaussian W it can only shave the top of the spectrum
    assert errs[-1] < (0.5 if precision == "nvfp4" else 0.95) * errs[0], errs


def test_subspace_iteration_matches_exact_svd_on_a_gapped_spectrum():
    """The subspace path (forced on a small matrix, with a given start
    block) recovers the top singular triplets of a matrix with a clear gap
    after r: singular values to 1e-10 and the rank-r product to 1e-9."""
    rng = np.random.default_rng(4)
    m, n, r = 300, 200, 8
    U0, _ = np.linalg.qr(rng.standard_normal((m, m)))
    V0, _ = np.linalg.qr(rng.standard_normal((n, n)))
    s0 = np.concatenate([np.linspace(50, 20, r), 0.5 * np.exp(-np.arange(n - r) / 40.0)])
    A = (U0[:, :n] * s0[None, :]) @ V0.T
    omega = rng.standard_normal((n, r + 8))
    U, s, V = S.truncated_svd(A, r, omega=omega)
    assert np.allclose(s, s0[:r], rtol=1e-10)
    Ue, se, Vte = np.linalg.svd(A, full_matrices=False)
    assert np.allclose((U * s) @ V.T, (Ue[:, :r] * se[:r]) @ Vte[:r], rtol=0, atol=1e-9 * s0[0])
    # the same start block through the seeded path gives the same result
    U2, s2, V2 = S.truncated_svd(A, r, oversample=8, seed=9, iterate=True)
    assert np.allclose(s2, s0[:r], rtol=1e-10)
