"""Run-to-run determinism at full size: the quantiser, the NVFP4 GEMM and the
INT4 GEMM, each called five times on the same inputs in the bench's launch
configuration, must give bit-identical outputs.  Their stage and scale
rings release shared memory back to the copy engine while other warps still
work on it, and the lora partials are reduced across CTAs; every order of
those steps is fixed, so no launch may differ from another in any bit."""
import pytest
import torch

import synth
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu

REPEATS = 5


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def _prepare_on_gpu(svdq, workload, seed, precision):
    """Weights prepared entirely on the GPU (lambda, factors, preparation), as
    the bench does: determinism needs no oracle."""
    li = synth.make_layer(workload, seed)
    M, K, N, r = li.shape.M, li.shape.K, li.shape.N, li.shape.rank
    X = T.dev_u16(li.x_bits)
    W = T.dev_f32(li.w)
    lam = torch.empty(K, dtype=torch.float32, device="cuda")
    svdq.svdq_smoothing_lambda(X, W, lam, torch.empty(2 * K, dtype=torch.float32, device="cuda"))
    L1 = torch.empty((r, K), dtype=torch.int16, device="cuda")
    L2 = torch.empty((N, r), dtype=torch.int16, device="cuda")
    omega = T.dev_f32(synth.svd_start_block(N, r + 16, seed))
    lr_ws = T.aligned_empty(svdq.svdq_lowrank_workspace_bytes(N, K))
    svdq.svdq_lowrank_factors(W, lam, r, omega, L1, L2, lr_ws)
    w = svdq.prepare_layer(W, lam, L1, L2, T.dev_u16(li.bias_bits), r, T.PREC[precision])
    gx = 1.0
    if precision == "nvfp4":
        g = torch.empty(1, dtype=torch.float32, device="cuda")
        svdq.svdq_act_global_scale(w, X, g)
        gx = float(g.item())
    return w, X, gx, M, K, N


@pytest.mark.parametrize("workload,seed,precision", [("qkv", 2, "nvfp4"), ("mlp_down", 3, "nvfp4"),
                                                     ("int4", 4, "int4")])
def test_repeated_calls_are_bit_identical(svdq, workload, seed, precision):
    w, X, gx, M, K, N = _prepare_on_gpu(svdq, workload, seed, precision)
    rp = w.view().rank_pad
    first = None
    for _ in range(REPEATS):
        qx = torch.empty(svdq.svdq_act_codes_bytes(w, M), dtype=torch.uint8, device="cuda")
        sx = T.aligned_empty(svdq.svdq_act_scale_bytes(w, M))
        la = torch.empty((M, rp), dtype=torch.float32, device="cuda")
        # poison the outputs: nothing may be left over from a previous call
        qx.fill_(0xA5)
        sx.fill_(0x5A)
        la.fill_(float("nan"))
        svdq.svdq_quantize_act_lora_down(w, X, M, gx, qx, sx, la)
        Y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        svdq.svdq_w4a4_gemm_lora_up(w, qx, sx, gx, la, M, Y, svdq.SVDQ_OUT_BF16)
        torch.cuda.synchronize()
        got = (qx.clone(), sx.clone(), la.clone(), Y.clone())
        if first is None:
            first = got
            assert bool(torch.isfinite(Y.float()).all())
        else:
            for a, b, what in zip(first, got, ("codes", "scales", "lora_act", "Y")):
                assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), what
    assert svdq.svdq_device_status(w) == 0
