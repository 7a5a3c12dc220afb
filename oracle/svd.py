"""Truncated SVD for the low-rank branch (oracle; test infrastructure).

The pages name the method "Singular Value Decomposition Quantization"
(ai2day, "Was ist Nunchaku Lite") and say that a small 16-bit low-rank
branch carries the hardest part of each weight matrix (Nunchaku 4-bit in
Diffusers, "Nunchaku und SVDQuant"), with rank 32 in the config block.  The
factorisation itself is not spelled out; the plain reading is the truncated
SVD of the smoothed weight: A = U S V^T, L1 = U_r S_r, L2 = V_r^T.

Small matrices use LAPACK's full SVD (numpy.linalg.svd).  Large ones use
block subspace iteration with a fixed seed (Halko, Martinsson & Tropp,
"Finding structure with randomness", 2011: a Gaussian start block, q power
steps with re-orthonormalisation, then a Rayleigh-Ritz step), which gives a
near-best rank-r factor; the layer's parity does not depend on the factor
being optimal, because L1 and L2 are inputs consumed identically by both
implementations.
"""
from __future__ import annotations

import numpy as np

EXACT_MAX_DIM = 1024


def truncated_svd(A: np.ndarray, r: int, power_steps: int = 4, oversample: int = 16, seed: int = 1234,
                  omega: np.ndarray | None = None, iterate: bool = False):
    """Return (U_r, s_r, V_r) of the fp64 matrix A (m x n): A ~ U_r diag(s_r) V_r^T.

    U_r is m x r, V_r is n x r, s_r is non-increasing.  `omega` (n x ell)
    replaces the seeded Gaussian start block of the subspace iteration, and
    `iterate` selects that iteration also for small matrices.
    """
    A = np.asarray(A, dtype=np.float64)
    m, n = A.shape
    r = int(r)
    if r == 0:
        return np.zeros((m, 0)), np.zeros(0), np.zeros((n, 0))
    if r > min(m, n):
        raise ValueError("rank larger than the matrix")
    if min(m, n) <= EXACT_MAX_DIM and not iterate and omega is None:
        U, s, Vt = np.linalg.svd(A, full_matrices=False)
        return U[:, :r], s[:r], Vt[:r].T
    if omega is None:
        rng = np.random.Generator(np.random.PCG64(seed))
        ell = min(r + oversample, min(m, n))
        omega = rng.standard_normal((n, ell))
    Q, _ = np.linalg.qr(A @ np.asarray(omega, dtype=np.float64))
    for _ in range(power_steps):
        Z, _ = np.linalg.qr(A.T @ Q)
        Q, _ = np.linalg.qr(A @ Z)
    B = Q.T @ A  # ell x n
    Ub, s, Vt = np.linalg.svd(B, full_matrices=False)
    U = Q @ Ub
    return U[:, :r], s[:r], Vt[:r].T
