"""Parity at the full workload sizes, in the launch configuration the bench
uses: every weight and activation code and scale bit-exact against the
oracle; Y checked on seeded sampled rows (rows are independent given the
codes, so the oracle computes only those rows)."""
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


@pytest.mark.parametrize("workload", ["qkv", "mlp_up", "mlp_down"])
def test_full_size_nvfp4(svdq, workload):
    li = synth.make_layer(workload, 2)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    h = T.weights_to_host(w)
    assert h["g_w"] == ol.prep.g_w
    assert np.array_equal(T.unpack_codes(h["qw"]), ol.prep.qw)
    assert np.array_equal(T.untile_nvfp4_scales(h["sw"], N, K), ol.prep.sw)

    X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
    rows = np.sort(np.random.default_rng(7).choice(M, SAMPLE_ROWS, replace=False))
    xs = li.x[rows]
    act = V.quantize_activations(xs, ol.prep, ol.gx)
    codes = T.unpack_codes(qx.cpu().numpy().reshape(M, K // 2))
    assert np.array_equal(codes[rows], act.qx)
    assert np.array_equal(T.untile_nvfp4_scales(sx.cpu().numpy(), M, K)[rows], act.sx)

    ref = V.forward_from_codes(act, ol.prep, ol.gx)
    rms = np.sqrt(np.mean(ref ** 2))
    for out_dtype in (1, 0):
        Y = torch.empty((M, N), dtype=torch.float32 if out_dtype else torch.bfloat16, device="cuda")
        svdq.svdq_w4a4_gemm_lora_up(w, qx, sx, float(ol.gx), la, M, Y, out_dtype)
        torch.cuda.synchronize()
        y = Y.float().cpu().numpy()[rows].astype(np.float64)
        d = y - ref
        assert np.linalg.norm(d) / np.linalg.norm(ref) <= REL_F
        if out_dtype:
            assert np.abs(d).max() <= MAX_ABS * rms
        else:
            half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
            assert np.all(np.abs(d) <= MAX_ABS * rms + half_ulp)
        assert np.all(np.isfinite(Y.float().cpu().numpy()))
    assert svdq.svdq_device_status(w) == 0


def test_full_size_int4(svdq):
    """The INT4 configuration (four images: 18432 x 3072 -> 3072, rank 32)
    at full size: every CTA of the persistent INT4 GEMM runs many tiles."""
    li = synth.make_layer("int4", 4)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    ol = T.oracle_layer(li, precision="int4")
    w = T.gpu_prepare(svdq, li, ol, "int4")
    h = T.weights_to_host(w)
    assert np.array_equal(T.unpack_codes(h["qw"]), (ol.prep.qw.astype(np.int16) & 0xF).astype(np.uint8))
    sw = h["sw"].view(np.float16).reshape(K // 64, h["n_pad"])[:, :N].T
    assert np.array_equal(sw.view(np.uint16), ol.prep.sw.view(np.uint16))

    X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, 1.0)
    rows = np.sort(np.random.default_rng(8).choice(M, SAMPLE_ROWS, replace=False))
    act = V.quantize_activations(li.x[rows], ol.prep)
    codes = T.nibbles_to_int(T.unpack_codes(qx.cpu().numpy().reshape(M, K // 2)))
    assert np.array_equal(codes[rows], act.qx)
    mp = (M + 127) // 128 * 128
    sxh = sx.cpu().numpy().view(np.float16).reshape(K // 64, mp)
    assert np.array_equal(sxh[:, rows].T.view(np.uint16), act.sx.view(np.uint16))

    ref = V.forward_from_codes(act, ol.prep)
    rms = np.sqrt(np.mean(ref ** 2))
    for out_dtype in (1, 0):
        Y = torch.empty((M, N), dtype=torch.float32 if out_dtype else torch.bfloat16, device="cuda")
        svdq.svdq_w4a4_gemm_lora_up(w, qx, sx, 1.0, la, M, Y, out_dtype)
        torch.cuda.synchronize()
        y = Y.float().cpu().numpy()[rows].astype(np.float64)
        d = y - ref
        assert np.linalg.norm(d) / np.linalg.norm(ref) <= REL_F
        if out_dtype:
            assert np.abs(d).max() <= MAX_ABS * rms
        else:
            half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
            assert np.all(np.abs(d) <= MAX_ABS * rms + half_ulp)
        assert np.all(np.isfinite(Y.float().cpu().numpy()))
    assert svdq.svdq_device_status(w) == 0


def test_stack_block_through_forward(svdq):
    """One block of the 57-block denoising stack at full size (QKV 3072 ->
    9216, out 3072 -> 3072, MLP up 3072 -> 12288, down 12288 -> 3072; M =
    4608, rank 32, NVFP4), every linear through svdq_linear_forward with the
    per-layer seeds of the stack: sampled codes and scales bit-exact, sampled
    Y rows within the bf16-output tolerance."""
    for layer, name in enumerate(synth.STACK_LAYERS):
        li = synth.make_layer(name, synth.stack_seed(0, layer))
        M, K, N = li.shape.M, li.shape.K, li.shape.N
        ol = T.oracle_layer(li)
        w = T.gpu_prepare(svdq, li, ol)
        rows = np.sort(np.random.default_rng(100 + layer).choice(M, 64, replace=False))
        act = V.quantize_activations(li.x[rows], ol.prep, ol.gx)
        X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
        codes = T.unpack_codes(qx.cpu().numpy().reshape(M, K // 2))
        assert np.array_equal(codes[rows], act.qx), name
        assert np.array_equal(T.untile_nvfp4_scales(sx.cpu().numpy(), M, K)[rows], act.sx), name
        ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        svdq.svdq_linear_forward(w, X, M, float(ol.gx), Y, ws, ws.numel(), 0)
        torch.cuda.synchronize()
        assert svdq.svdq_device_status(w) == 0
        ref = V.forward_from_codes(act, ol.prep, ol.gx)
        y = Y.float().cpu().numpy()[rows].astype(np.float64)
        d = y - ref
        rms = np.sqrt(np.mean(ref ** 2))
        assert np.linalg.norm(d) / np.linalg.norm(ref) <= REL_F, name
        half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
        assert np.all(np.abs(d) <= MAX_ABS * rms + half_ulp), name


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
            r_ = ref[:, sec * wd:(sec + 1) * wd]
            d = y[:, sec * wd:(sec + 1) * wd] - r_
            rms = np.sqrt(np.mean(r_ ** 2))
            assert np.linalg.norm(d) / np.linalg.norm(r_) <= REL_F
            if out_dtype:
                assert np.abs(d).max() <= MAX_ABS * rms
            else:
                half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(r_), 1e-30))) - 8)
                assert np.all(np.abs(d) <= MAX_ABS * rms + half_ulp)
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
    y = Ya.float().cpu().numpy()[rows].astype(np.float64)
    d = y - ref
    rms = np.sqrt(np.mean(ystar ** 2))
    assert np.linalg.norm(d) <= 1.13 * REL_F * np.linalg.norm(ystar)
    half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
    assert np.all(np.abs(d) <= 1.13 * MAX_ABS * rms + half_ulp)
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
