"""Parity at the full workload sizes, in the launch configuration the bench
uses: every weight part and every activation code and scale of every row
bit-exact against the oracle (weights and scales exported in canonical
layout through the C ABI); Y checked on seeded sampled rows (rows are
independent given the codes, so the oracle computes only those rows)."""
import numpy as np
import pytest
import torch

import synth
from oracle import svdq as V
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu

REL_F = 2e-3
MAX_ABS = 1e-2
SAMPLE_ROWS = 96


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def _rows_of(act: V.ActQuant, rows) -> V.ActQuant:
    return V.ActQuant(act.qx[rows], act.sx[rows], act.lora_act[rows])


@pytest.mark.parametrize("workload,seed,precision", [("qkv", 2, "nvfp4"), ("mlp_up", 2, "nvfp4"),
                                                     ("mlp_down", 3, "nvfp4"), ("int4", 4, "int4")])
def test_full_size(svdq, workload, seed, precision):
    """The FLUX fused QKV projection, both MLP linears and the INT4 batch of
    four images: all weight parts and all activation codes and scales
    bit-exact; Y on sampled rows in both output types."""
    li = synth.make_layer(workload, seed)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    ol = T.oracle_layer(li, precision=precision)
    w = T.gpu_prepare(svdq, li, ol, precision)
    T.check_weights_exact(svdq, w, T.expected_weights(li, ol.prep))

    X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
    exp = T.check_act_exact(svdq, w, li.x, ol, qx, sx, la)
    rows = np.sort(np.random.default_rng(7).choice(M, SAMPLE_ROWS, replace=False))
    ref = V.forward_from_codes(_rows_of(exp["act"], rows), ol.prep, ol.gx if precision == "nvfp4" else None)
    for out_dtype in (1, 0):
        Y = torch.empty((M, N), dtype=torch.float32 if out_dtype else torch.bfloat16, device="cuda")
        svdq.svdq_w4a4_gemm_lora_up(w, qx, sx, float(ol.gx), la, M, Y, out_dtype)
        torch.cuda.synchronize()
        T.check_y(Y[torch.from_numpy(rows).cuda()].float().cpu().numpy(), ref, out_dtype, REL_F, MAX_ABS)
        assert bool(torch.isfinite(Y.float()).all())
    assert svdq.svdq_device_status(w) == 0


def test_full_size_qkv_prologue(svdq):
    """The fused QKV projection (M=4608, K=3072, N=9216 = 3 x 24 heads x
    128, rank 32, NVFP4) with the attention prologue in the GEMM epilogue:
    sampled rows of Q', K', V against the oracle's prologue applied to the
    fp64 layer output."""
    from oracle import qkv as A
    li = synth.make_layer("qkv", 2)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    heads = N // 384
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
    nq, nk, cs, sn = synth.qkv_prologue_inputs(M, 128, 29)
    dq, dk, dc, ds = T.dev_f32(nq), T.dev_f32(nk), T.dev_f32(cs.T.copy()), T.dev_f32(sn.T.copy())
    pro = svdq.make_qkv_prologue(heads, dq, dk, dc, ds, 1e-6)
    rows = np.sort(np.random.default_rng(9).choice(M, SAMPLE_ROWS, replace=False))
    act = V.quantize_activations(li.x[rows], ol.prep, ol.gx)
    ref = A.qkv_prologue(V.forward_from_codes(act, ol.prep, ol.gx), heads, 128, nq, nk, cs[rows], sn[rows], 1e-6)
    wd = heads * 128
    for out_dtype in (1, 0):
        Y = torch.empty((M, N), dtype=torch.float32 if out_dtype else torch.bfloat16, device="cuda")
        svdq.svdq_w4a4_gemm_lora_up_qkv(w, qx, sx, float(ol.gx), la, M, pro, Y, out_dtype)
        torch.cuda.synchronize()
        y = Y.float().cpu().numpy()[rows].astype(np.float64)
        for sec in range(3):
            T.check_y(y[:, sec * wd:(sec + 1) * wd], ref[:, sec * wd:(sec + 1) * wd], out_dtype, REL_F, MAX_ABS)
    assert svdq.svdq_device_status(w) == 0


def test_full_size_mlp_chain(svdq):
    """The FLUX feed-forward at full size (M=4608; up 3072 -> 12288, GELU,
    down 12288 -> 3072; rank 32, NVFP4) with the dynamic tensor scale: the
    up-projection's epilogue applies the GELU and max-reduces the down
    layer's amax.  Sampled up rows against the oracle (the GELU widens the
    bound by its Lipschitz constant 1.13); the amax word equal to the
    separate amax pass over the stored output; the down layer on that
    output, with the word as its scale, equal to the static layer."""
    from oracle import chain as C
    li_a = synth.make_layer("mlp_up", 2)
    li_b = synth.make_layer("mlp_down", 3)
    M, K, N = li_a.shape.M, li_a.shape.K, li_a.shape.N
    ol_a = T.oracle_layer(li_a)
    ol_b = T.oracle_layer(li_b)
    wa = T.gpu_prepare(svdq, li_a, ol_a)
    wb = T.gpu_prepare(svdq, li_b, ol_b)
    words = torch.full((2,), 1e30, dtype=torch.float32, device="cuda")
    il_b = T.dev_f32(ol_b.prep.inv_lam)
    epi = svdq.make_epilogue_next(svdq.SVDQ_ACT_GELU_TANH, il_b, words[1:])
    ws = T.aligned_empty(max(svdq.svdq_workspace_bytes(wa, M), svdq.svdq_workspace_bytes(wb, M)))
    Ya = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    svdq.svdq_linear_forward_dyn(wa, T.dev_u16(li_a.x_bits), M, None, Ya, ws, ws.numel(), epi=epi)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(wa) == 0
    rows = np.sort(np.random.default_rng(13).choice(M, SAMPLE_ROWS, replace=False))
    act = V.quantize_activations(li_a.x[rows], ol_a.prep, ol_a.gx)  # ol_a.gx: the dynamic scale of all of X
    ystar = V.forward_from_codes(act, ol_a.prep, ol_a.gx)
    ref = C.gelu_tanh(ystar)
    T.check_y(Ya.float().cpu().numpy()[rows], ref, 0, REL_F, MAX_ABS, widen=1.13, ref_for_scale=ystar)
    a2 = torch.empty(1, dtype=torch.float32, device="cuda")
    svdq.svdq_act_amax(wb, Ya.view(torch.int16), a2)
    amax = np.float32(words[1].item())
    assert np.float32(a2.item()) == amax and amax > 0
    Yb = torch.empty((M, li_b.shape.N), dtype=torch.bfloat16, device="cuda")
    svdq.svdq_linear_forward_dyn(wb, Ya.view(torch.int16), M, words[1:], Yb, ws, ws.numel())
    Yb2 = torch.empty_like(Yb)
    svdq.svdq_linear_forward(wb, Ya.view(torch.int16), M, float(np.float32(amax / np.float32(2688.0))), Yb2, ws,
                             ws.numel(), 0)
    torch.cuda.synchronize()
    assert torch.equal(Yb, Yb2)
    assert svdq.svdq_device_status(wb) == 0
