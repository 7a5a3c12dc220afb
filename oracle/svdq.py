"""The SVDQuant W4A4 linear layer, step by step (oracle; test infrastructure).

What the layer computes (Nunchaku 4-bit in Diffusers, "Nunchaku und
SVDQuant"; charmloop.ai news item, second paragraph):

    X_hat = X / lambda                      (outliers migrate into the weights)
    W_til = W * diag(lambda)                (so X_hat W_til^T = X W^T)
    W_til^T ~ L1 L2                         (16-bit low-rank branch, rank r)
    R     = W_til - (L1 L2)^T               (residual, quantised to 4 bits)
    Y     = X_hat L1 L2 + Q(X_hat) Q(R)^T + b

with the lora-down X_hat L1 computed next to the activation quantisation and
the lora-up added inside the 4-bit GEMM.

Shapes and storage (PyTorch nn.Linear orientation): X is M x K (bf16),
W is N x K (fp32), lambda is K (fp32), L1 is stored r x K (bf16), L2 is
stored N x r (bf16), b is N (bf16), Y is M x N.

Readings of steps the pages leave open (listed again in the design notes):
  * lambda_k = sqrt(max_m |X[m,k]| / max_n |W[n,k]|) in fp64, rounded to
    fp32; lambda_k = 1 when either maximum is 0.  Calibration uses the same X.
  * inv_lambda_k = RN32(1 / lambda_k); X_hat = RN32(X * inv_lambda).
  * W_til = RN32(W * lambda).
  * L1 = bf16(U_r S_r)^T and L2 = bf16(V_r) from the truncated SVD of W_til^T.
  * R[n,k] = RN32 of the fp64 chain acc = W_til[n,k]; acc -= L1[t,k]*L2[n,t]
    for t = 0..r-1 in order (each product of two bf16 values is exact in fp64,
    so every step is one fp64 rounding).
  * The lora-down uses L1s[t,k] = bf16(RN32(L1[t,k] * inv_lambda_k)) against
    the unsmoothed bf16 X, so that X_hat L1 = X L1s up to that rounding.
  * Quantisers: see oracle.quant.
  * The activation tensor scale g_x is an input of each call (static
    calibration); calibration sets it from amax |X_hat| by the tensor-scale
    rule.
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import formats as F
from . import quant as Q
from .svd import truncated_svd


def smoothing_lambda(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    """Per-input-channel smoothing factor lambda (K,) in fp32."""
    # maxima of magnitudes are exact in the inputs' own type; ratio and root in fp64
    ax = np.max(np.abs(np.asarray(x)), axis=0).astype(np.float64)
    aw = np.max(np.abs(np.asarray(w)), axis=0).astype(np.float64)
    with np.errstate(divide="ignore", invalid="ignore"):
        lam = np.sqrt(ax / aw)
    lam = np.where((ax == 0) | (aw == 0), 1.0, lam)
    return lam.astype(np.float32)


def inv_lambda(lam: np.ndarray) -> np.ndarray:
    return np.float32(1.0) / np.asarray(lam, dtype=np.float32)


def smooth_weight(w: np.ndarray, lam: np.ndarray) -> np.ndarray:
    """W_til = RN32(W * lambda) (N x K fp32)."""
    return np.asarray(w, dtype=np.float32) * np.asarray(lam, dtype=np.float32)[None, :]


def smooth_activation(x: np.ndarray, inv_lam: np.ndarray) -> np.ndarray:
    """X_hat = RN32(X * inv_lambda) (M x K fp32)."""
    return np.asarray(x, dtype=np.float32) * np.asarray(inv_lam, dtype=np.float32)[None, :]


def lowrank_factors(w: np.ndarray, lam: np.ndarray, rank: int, omega: np.ndarray | None = None,
                    power_steps: int = 4):
    """(L1 stored r x K, L2 stored N x r), both bf16 values held in fp32.
    With `omega` (N x ell) the subspace iteration starts from that block."""
    wt = smooth_weight(w, lam).astype(np.float64)  # N x K
    U, s, V = truncated_svd(wt.T, rank, power_steps=power_steps, omega=omega)  # wt^T = U S V^T
    L1 = F.bf16_rn((U * s[None, :]).T).astype(np.float32)  # r x K
    L2 = F.bf16_rn(V).astype(np.float32)  # N x r
    return L1, L2


def residual(wt: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """R = RN32(fp64 chain W_til - sum_t L1[t,:] L2[:,t]) in fixed t order."""
    wt = np.asarray(wt, dtype=np.float32)
    L1d = np.asarray(L1, dtype=np.float64)
    L2d = np.asarray(L2, dtype=np.float64)
    out = np.empty(wt.shape, np.float32)
    B = 64  # rows per block: the chain of each element is the same, blocks only keep it in cache
    for i in range(0, wt.shape[0], B):
        acc = wt[i:i + B].astype(np.float64)
        tmp = np.empty_like(acc)
        for t in range(L1d.shape[0]):
            np.multiply(L2d[i:i + B, t:t + 1], L1d[t:t + 1, :], out=tmp)  # exact: two bf16 values
            acc -= tmp
        out[i:i + B] = acc
    return out


@dataclasses.dataclass
class Prepared:
    precision: str  # "nvfp4" | "int4"
    K: int
    N: int
    rank: int
    lam: np.ndarray  # K fp32
    inv_lam: np.ndarray  # K fp32
    L1: np.ndarray  # r x K (bf16 values)
    L2: np.ndarray  # N x r (bf16 values)
    L1s: np.ndarray  # r x K (bf16 values)
    bias: np.ndarray  # N (bf16 values, fp32)
    R: np.ndarray  # N x K fp32
    g_w: np.float32  # NVFP4 tensor scale (1 for INT4)
    qw: np.ndarray  # N x K codes: E2M1 nibbles (nvfp4) or int8 in [-8, 7] (int4)
    sw: np.ndarray  # N x K/16 E4M3 bytes (nvfp4) or N x K/64 float16 (int4)


def prepare_weights(w, lam, L1, L2, bias, precision: str = "nvfp4") -> Prepared:
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    L1 = np.asarray(L1, dtype=np.float32).reshape(-1, K)
    L2 = np.asarray(L2, dtype=np.float32).reshape(N, -1)
    r = L1.shape[0]
    lam = np.asarray(lam, dtype=np.float32)
    il = inv_lambda(lam)
    wt = smooth_weight(w, lam)
    R = residual(wt, L1, L2)
    L1s = F.bf16_rn(L1 * il[None, :]).astype(np.float32)  # fp32 product, then bf16
    if bias is None:
        bias = np.zeros(N, dtype=np.float32)
    if precision == "nvfp4":
        g_w = Q.nvfp4_tensor_scale(np.max(np.abs(R)) if R.size else 0.0)
        qw, sw = Q.nvfp4_quantize(R, g_w)
    elif precision == "int4":
        g_w = np.float32(1.0)
        qw, sw = Q.int4_quantize(R)
    else:
        raise ValueError(precision)
    return Prepared(precision, K, N, r, lam, il, L1, L2, L1s, np.asarray(bias, np.float32), R, g_w, qw, sw)


def act_global_scale(x: np.ndarray, inv_lam: np.ndarray) -> np.float32:
    """Static activation tensor scale g_x = RN32(amax |X_hat| / 2688)."""
    xh = smooth_activation(x, inv_lam)
    return Q.nvfp4_tensor_scale(np.max(np.abs(xh)) if xh.size else 0.0)


@dataclasses.dataclass
class ActQuant:
    qx: np.ndarray  # M x K codes (nibbles or int8)
    sx: np.ndarray  # M x K/16 E4M3 bytes or M x K/64 float16
    lora_act: np.ndarray  # M x r fp64: X L1s^T


def quantize_activations(x, prep: Prepared, g_x=None) -> ActQuant:
    """Smoothing + 4-bit quantisation of X_hat + lora-down X L1s^T.  NVFP4
    with g_x None: the dynamic tensor scale of this very X."""
    xh = smooth_activation(x, prep.inv_lam)
    if prep.precision == "nvfp4":
        if g_x is None:
            g_x = act_global_scale(x, prep.inv_lam)
        qx, sx = Q.nvfp4_quantize(xh, np.float32(g_x))
    else:
        qx, sx = Q.int4_quantize(xh)
    lora = np.asarray(x, dtype=np.float64) @ prep.L1s.astype(np.float64).T
    return ActQuant(qx, sx, lora)


def gemm_unscaled(a: ActQuant, prep: Prepared) -> np.ndarray:
    """The 4-bit product without tensor scales, in fp64:
    NVFP4: sum_b s_x s_w sum_{k in b} e2m1(qx) e2m1(qw);
    INT4:  sum_g s_x s_w sum_{k in g} qx qw."""
    if prep.precision == "nvfp4":
        dx = Q.nvfp4_dequantize(a.qx, a.sx, 1.0)
        dw = Q.nvfp4_dequantize(prep.qw, prep.sw, 1.0)
    else:
        dx = Q.int4_dequantize(a.qx, a.sx)
        dw = Q.int4_dequantize(prep.qw, prep.sw)
    return dx @ dw.T


def forward_from_codes(a: ActQuant, prep: Prepared, g_x=None) -> np.ndarray:
    """Y* = g_x g_w (4-bit product) + (X L1s^T) L2^T + b, in fp64.  NVFP4
    needs the tensor scale the codes were made with."""
    if prep.precision == "nvfp4" and g_x is None:
        raise ValueError("NVFP4 codes need their tensor scale g_x")
    S = gemm_unscaled(a, prep)
    if prep.precision == "nvfp4":
        S = S * (float(np.float32(g_x)) * float(prep.g_w))
    lora = a.lora_act @ prep.L2.astype(np.float64).T
    return S + lora + prep.bias.astype(np.float64)[None, :]


def forward(x, prep: Prepared, g_x=None) -> np.ndarray:
    """The layer in fp64; NVFP4 with g_x None takes the dynamic tensor
    scale of this X."""
    if g_x is None and prep.precision == "nvfp4":
        g_x = act_global_scale(x, prep.inv_lam)
    return forward_from_codes(quantize_activations(x, prep, g_x), prep, g_x)


def reference_dense(x, w, bias) -> np.ndarray:
    """The unquantised layer X W^T + b in fp64 (for quality invariants)."""
    out = np.asarray(x, np.float64) @ np.asarray(w, np.float64).T
    if bias is not None:
        out = out + np.asarray(bias, np.float64)[None, :]
    return out
