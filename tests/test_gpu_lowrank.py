"""The GPU truncated SVD (svdq_lowrank_factors) against the oracle's
subspace iteration started from the same block: singular values, the
quality of the rank-r approximation, orthonormal factors, and the rank-r
product on a spectrum with a gap."""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import svd as S
from oracle import svdq as V
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def _gpu_factors(svdq, w, lam, rank, omega, power_steps=4):
    N, K = w.shape
    ell = omega.shape[1]
    W = T.dev_f32(w)
    L = T.dev_f32(lam)
    O = T.dev_f32(omega)
    L1 = torch.empty((rank, K), dtype=torch.int16, device="cuda")
    L2 = torch.empty((N, rank), dtype=torch.int16, device="cuda")
    ws = T.aligned_empty(svdq.svdq_lowrank_workspace_bytes(N, K))
    svdq.svdq_lowrank_factors(W, L, rank, O, L1, L2, ws, oversample=ell - rank, power_steps=power_steps)
    torch.cuda.synchronize()
    f = lambda t: synth.f32_from_bf16_bits(t.cpu().numpy().view(np.uint16)).astype(np.float64)
    return f(L1), f(L2)


def _checks(w, lam, L1, L2, rank, omega, power_steps=4, s_rtol=2e-3, q_rtol=2e-3):
    wt = V.smooth_weight(w, lam).astype(np.float64)  # N x K
    U, s, Vv = S.truncated_svd(wt.T, rank, power_steps=power_steps, omega=omega.astype(np.float64))
    # singular values: the row norms of L1 (U has orthonormal columns)
    s_gpu = np.linalg.norm(L1, axis=1)
    assert np.allclose(s_gpu, s, rtol=s_rtol, atol=0), np.max(np.abs(s_gpu / s - 1))
    # orthonormal right factor (bf16-rounded)
    assert np.abs(L2.T @ L2 - np.eye(rank)).max() < 0.02
    # quality of the rank-r approximation: as good as the oracle's own factors
    L1o = F.bf16_rn((U * s[None, :]).T)
    L2o = F.bf16_rn(Vv)
    e_gpu = np.linalg.norm(wt - L2 @ L1)
    e_or = np.linalg.norm(wt - L2o @ L1o)
    assert e_gpu <= e_or * (1 + q_rtol), (e_gpu, e_or)
    return U, s, Vv


@pytest.mark.parametrize("workload,over,rank,ell", [
    ("qkv", dict(N=1536, K=1280), 32, 48),      # rank-4 spike plus a flat Gaussian part
    ("mlp_down", dict(N=768, K=2048), 16, 24),  # flat spectrum
    ("stack_out", dict(N=384, K=640), 64, 64),  # the largest subspace
])
def test_lowrank_against_oracle_iteration(svdq, workload, over, rank, ell):
    li = synth.make_layer(workload, 21, **over)
    lam = V.smoothing_lambda(li.x, li.w)
    omega = synth.svd_start_block(li.shape.N, ell, 21)
    L1, L2 = _gpu_factors(svdq, li.w, lam, rank, omega)
    _checks(li.w, lam, L1, L2, rank, omega)


def test_lowrank_gapped_spectrum_product(svdq):
    """With a gap after r the rank-r product is well defined: the GPU's
    equals the oracle's up to the bf16 rounding of the factors."""
    rng = np.random.default_rng(6)
    N, K, r, ell = 640, 512, 16, 32
    Uo, _ = np.linalg.qr(rng.standard_normal((N, N)))
    Vo, _ = np.linalg.qr(rng.standard_normal((K, K)))
    s0 = np.concatenate([np.linspace(40, 10, r), 0.2 * np.exp(-np.arange(K - r) / 50.0)])
    w = ((Uo[:, :K] * s0[None, :]) @ Vo.T).astype(np.float32)
    lam = np.ones(K, np.float32)
    omega = synth.svd_start_block(N, ell, 6)
    L1, L2 = _gpu_factors(svdq, w, lam, r, omega)
    U, s, Vv = _checks(w, lam, L1, L2, r, omega)
    P_or = (Vv * s[None, :]) @ U.T  # N x K
    assert np.linalg.norm(L2 @ L1 - P_or) / np.linalg.norm(P_or) < 1e-2


def test_lowrank_full_size_qkv(svdq):
    """The FLUX QKV projection at full size (9216 x 3072, rank 32, 16
    oversampling, 4 power steps), as weight preparation uses it."""
    li = synth.make_layer("qkv", 2)
    lam = V.smoothing_lambda(li.x, li.w)
    omega = synth.svd_start_block(li.shape.N, 48, 2)
    L1, L2 = _gpu_factors(svdq, li.w, lam, 32, omega)
    _checks(li.w, lam, L1, L2, 32, omega)


def test_lowrank_argument_errors(svdq):
    lib = svdq.load_library()
    t = torch.zeros(4096, dtype=torch.float32, device="cuda")
    ws = T.aligned_empty(svdq.svdq_lowrank_workspace_bytes(64, 64))
    args = lambda rank, over, steps, N=64, K=64, wsb=ws.numel(): lib.svdq_lowrank_factors(
        t.data_ptr(), N, K, t.data_ptr(), rank, over, steps, t.data_ptr(), t.data_ptr(), t.data_ptr(), ws.data_ptr(),
        wsb, None)
    assert args(12, 4, 2) == 2    # rank % 8
    assert args(64, 8, 2) == 2    # ell > 64
    assert args(16, 8, 17) == 2   # too many power steps
    assert args(16, 8, 2, N=16) == 2  # ell > N
    assert args(16, 8, 2, wsb=16) == 7  # workspace too small
    assert lib.svdq_lowrank_factors(None, 64, 64, t.data_ptr(), 16, 8, 2, t.data_ptr(), t.data_ptr(), t.data_ptr(),
                                    ws.data_ptr(), ws.numel(), None) == 1
    assert args(16, 8, 2) == 0
    torch.cuda.synchronize()
