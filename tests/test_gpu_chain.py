"""GPU parity of the dynamic activation tensor scale and of chained layers
(the epilogue's GELU and its max-reduction of the next layer's amax),
through the C ABI, against the oracle on the same seeded inputs.

Tolerances: Y as in the single-layer parity tests; after the GELU the bound
grows by the GELU's Lipschitz constant (max slope of the tanh form 1.1290,
so 1.13), since the activation is applied to the fp32 layer output whose
error those bounds cover.  Integer and byte results (codes, scales, the amax
words, which are maxima of values both sides round the same way) are
compared bit for bit."""
import numpy as np
import pytest
import torch

import synth
from oracle import chain as C
from oracle import svdq as V
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu

REL_F = 2e-3
MAX_ABS = 1e-2
LIP = 1.13

# (name, layer a overrides, layer b overrides): layer b's K is layer a's N;
# ragged M, N not a multiple of the 256-wide tile, more tiles than CTAs
CHAIN_CASES = [
    ("small", dict(M=300, K=512, N=768), dict(K=768, N=512)),
    ("ragged", dict(M=129, K=320, N=320), dict(K=320, N=144)),
    ("many_tiles", dict(M=1100, K=256, N=2560), dict(K=2560, N=320)),
]


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def _pair(name, a_over, b_over, seed=21):
    li_a = synth.make_layer("mlp_up", seed, **a_over)
    li_b = synth.make_layer("mlp_down", seed + 1, M=a_over["M"], **b_over)
    return li_a, li_b


def _assert_close(y, ref, out_dtype, lip=1.0, rms_in=None):
    """y (GPU, stored) against ref (fp64): relative Frobenius and per-element
    bounds of the single-layer tests, scaled by `lip` for an activation."""
    rms = np.sqrt(np.mean(ref ** 2)) if rms_in is None else rms_in
    d = y.astype(np.float64) - ref
    assert np.linalg.norm(d) <= lip * REL_F * max(np.linalg.norm(ref), rms * np.sqrt(ref.size)), \
        float(np.linalg.norm(d) / np.linalg.norm(ref))
    bound = lip * MAX_ABS * rms
    if out_dtype == 0:
        bound = bound + 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
    assert np.all(np.abs(d) <= bound), float(np.max(np.abs(d) - bound))


def _ws(svdq, w, M):
    return T.aligned_empty(svdq.svdq_workspace_bytes(w, M))


def _ydev(M, N, out_dtype):
    return torch.empty((M, N), dtype=torch.float32 if out_dtype else torch.bfloat16, device="cuda")


def test_act_amax_bit_exact(svdq):
    li = synth.make_layer("qkv", 11, M=300, K=1024, N=768)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    a = torch.full((1,), 123.0, dtype=torch.float32, device="cuda")  # the call zeroes it first
    svdq.svdq_act_amax(w, T.dev_u16(li.x_bits), a)
    got = np.float32(a.item())
    assert got == C.act_amax(li.x, ol.prep.inv_lam)
    assert np.float32(got / np.float32(2688.0)) == ol.gx


@pytest.mark.parametrize("name,a_over,b_over", CHAIN_CASES, ids=[c[0] for c in CHAIN_CASES])
def test_dyn_quantize_bit_exact(svdq, name, a_over, b_over):
    li, _ = _pair(name, a_over, b_over)
    ol = T.oracle_layer(li)  # ol.gx: the oracle's dynamic scale of this X
    w = T.gpu_prepare(svdq, li, ol)
    M, K = li.shape.M, li.shape.K
    X = T.dev_u16(li.x_bits)
    a = torch.empty(1, dtype=torch.float32, device="cuda")
    svdq.svdq_act_amax(w, X, a)
    qx = T.aligned_empty(svdq.svdq_act_codes_bytes(w, M))
    sx = T.aligned_empty(svdq.svdq_act_scale_bytes(w, M))
    rp = w.view().rank_pad
    la = torch.empty((M, rp), dtype=torch.float32, device="cuda")
    svdq.svdq_quantize_act_lora_down_dyn(w, X, M, a, qx, sx, la)
    torch.cuda.synchronize()
    act = V.quantize_activations(li.x, ol.prep, ol.gx)
    assert np.array_equal(T.unpack_codes(qx[:M * K // 2].cpu().numpy().reshape(M, K // 2)), act.qx)
    assert np.array_equal(T.untile_nvfp4_scales(sx.cpu().numpy(), M, K), act.sx)
    # lora_act: the same buffer as the static call with the same g_x (bit for bit)
    X2, qx2, sx2, la2 = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
    assert torch.equal(la, la2) and torch.equal(qx, qx2) and torch.equal(sx, sx2)
    assert svdq.svdq_device_status(w) == 0


@pytest.mark.parametrize("out_dtype", [1, 0], ids=["f32", "bf16"])
@pytest.mark.parametrize("name,a_over,b_over", CHAIN_CASES, ids=[c[0] for c in CHAIN_CASES])
def test_dyn_forward_parity(svdq, name, a_over, b_over, out_dtype):
    li, _ = _pair(name, a_over, b_over)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M, N = li.shape.M, li.shape.N
    X = T.dev_u16(li.x_bits)
    ws = _ws(svdq, w, M)
    Yd = _ydev(M, N, out_dtype)
    svdq.svdq_linear_forward_dyn(w, X, M, None, Yd, ws, ws.numel(), out_dtype=out_dtype)
    Ys = _ydev(M, N, out_dtype)
    svdq.svdq_linear_forward(w, X, M, float(ol.gx), Ys, ws, ws.numel(), out_dtype)
    torch.cuda.synchronize()
    assert torch.equal(Yd, Ys)  # the in-kernel scale is the host's, bit for bit
    _assert_close(Yd.float().cpu().numpy(), V.forward(li.x, ol.prep, ol.gx), out_dtype)
    assert svdq.svdq_device_status(w) == 0


@pytest.mark.parametrize("activation", ["gelu_tanh", "none"])
@pytest.mark.parametrize("out_dtype", [0, 1], ids=["bf16", "f32"])
@pytest.mark.parametrize("name,a_over,b_over", CHAIN_CASES, ids=[c[0] for c in CHAIN_CASES])
def test_chain_epilogue(svdq, name, a_over, b_over, out_dtype, activation):
    li_a, li_b = _pair(name, a_over, b_over)
    ol_a = T.oracle_layer(li_a)
    ol_b = T.oracle_layer(li_b)  # layer b calibrated on its own seeded input
    wa = T.gpu_prepare(svdq, li_a, ol_a)
    wb = T.gpu_prepare(svdq, li_b, ol_b)
    M, N = li_a.shape.M, li_a.shape.N
    il_b = T.dev_f32(ol_b.prep.inv_lam)
    words = torch.full((2,), 1e30, dtype=torch.float32, device="cuda")  # stale values: the forward zeroes its word
    act = svdq.SVDQ_ACT_GELU_TANH if activation == "gelu_tanh" else svdq.SVDQ_ACT_NONE
    epi = svdq.make_epilogue_next(act, il_b, words[1:])
    ws = _ws(svdq, wa, M)
    Ya = _ydev(M, N, out_dtype)
    svdq.svdq_linear_forward_dyn(wa, T.dev_u16(li_a.x_bits), M, None, Ya, ws, ws.numel(), epi=epi,
                                 out_dtype=out_dtype)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(wa) == 0
    ya = Ya.float().cpu().numpy()
    amax = np.float32(words[1].item())

    # layer a's stored output against the oracle
    ystar = V.forward(li_a.x, ol_a.prep, ol_a.gx)
    ref = C.ACTIVATIONS[activation](ystar)
    lip = LIP if activation == "gelu_tanh" else 1.0
    _assert_close(ya, ref, out_dtype, lip=lip, rms_in=np.sqrt(np.mean(ystar ** 2)))

    # the word is the max of |RN32(y_stored * 1/lambda_b)| over the stored output
    ilh = ol_b.prep.inv_lam.astype(np.float32)
    assert amax == np.max(np.abs(ya.astype(np.float32) * ilh[None, :]))
    if out_dtype == 0:
        a2 = torch.empty(1, dtype=torch.float32, device="cuda")
        svdq.svdq_act_amax(wb, Ya.view(torch.int16), a2)  # the separate amax pass over the same Y
        assert np.float32(a2.item()) == amax
    # and close to the oracle's amax of its own stored output
    amax_ref = C.act_amax(C.round_output(ref, "bf16" if out_dtype == 0 else "f32"), ol_b.prep.inv_lam)
    slack = float(ilh.max()) * lip * MAX_ABS * np.sqrt(np.mean(ystar ** 2)) + 2.0 ** -7 * float(amax_ref)
    assert abs(float(amax) - float(amax_ref)) <= slack

    if out_dtype == 0:
        # layer b on that output with the word as its dynamic scale equals
        # the static layer given g_x = RN32(amax / 2688), bit for bit
        Mb, Nb = M, li_b.shape.N
        wsb = _ws(svdq, wb, Mb)
        Yb = _ydev(Mb, Nb, 0)
        svdq.svdq_linear_forward_dyn(wb, Ya.view(torch.int16), Mb, words[1:], Yb, wsb, wsb.numel())
        Yb2 = _ydev(Mb, Nb, 0)
        g_b = np.float32(amax / np.float32(2688.0)) if amax != 0 else np.float32(1.0)  # the header's rule
        svdq.svdq_linear_forward(wb, Ya.view(torch.int16), Mb, float(g_b), Yb2, wsb, wsb.numel(), 0)
        torch.cuda.synchronize()
        assert torch.equal(Yb, Yb2)
        assert svdq.svdq_device_status(wb) == 0
        # end to end against the oracle's chain: the two sides quantise
        # inputs that differ by output rounding, so this bounds gross errors
        # (a wrong scale, activation or factor) rather than rounding
        if activation == "gelu_tanh":
            _, amax_o, yb_ref = C.chain_forward(li_a.x, ol_a.prep, ol_b.prep, "gelu_tanh", "bf16")
            yb = Yb.float().cpu().numpy().astype(np.float64)
            assert np.linalg.norm(yb - yb_ref) <= 5e-2 * np.linalg.norm(yb_ref)


def test_zero_input_takes_unit_scale(svdq):
    li = synth.make_layer("mlp_up", 3, M=130, K=256, N=256)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M, N = 130, 256
    X = torch.zeros((M, 256), dtype=torch.int16, device="cuda")
    ws = _ws(svdq, w, M)
    Y = _ydev(M, N, 1)
    svdq.svdq_linear_forward_dyn(w, X, M, None, Y, ws, ws.numel(), out_dtype=1)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w) == 0
    assert np.array_equal(Y.cpu().numpy(), np.broadcast_to(li.bias, (M, N)))


def test_nonfinite_dynamic_scale_sets_status(svdq):
    li = synth.make_layer("mlp_up", 4, M=64, K=256, N=256)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M, K = 64, 256
    a = torch.full((1,), float("inf"), dtype=torch.float32, device="cuda")
    qx = T.aligned_empty(svdq.svdq_act_codes_bytes(w, M))
    sx = T.aligned_empty(svdq.svdq_act_scale_bytes(w, M))
    la = torch.empty((M, w.view().rank_pad), dtype=torch.float32, device="cuda")
    svdq.svdq_quantize_act_lora_down_dyn(w, T.dev_u16(li.x_bits), M, a, qx, sx, la)
    assert svdq.svdq_device_status(w) == 1  # SVDQ_ERR_INVALID_ARG, then cleared
    assert svdq.svdq_device_status(w) == 0


def test_chain_argument_errors(svdq):
    li = synth.make_layer("mlp_up", 5, M=64, K=256, N=256)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    w4 = T.gpu_prepare(svdq, li, T.oracle_layer(li, precision="int4"), "int4")
    M = 64
    X = T.dev_u16(li.x_bits)
    ws = _ws(svdq, w, M)
    Y = _ydev(M, 256, 0)
    il = T.dev_f32(ol.prep.inv_lam)
    word = torch.zeros(2, dtype=torch.float32, device="cuda")
    lib = svdq.load_library()

    def fwd(wt, x_amax, epi, pro=None):
        return lib.svdq_linear_forward_dyn(wt.handle, X.data_ptr(), M, x_amax, pro, epi, Y.data_ptr(), 0,
                                           ws.data_ptr(), ws.numel(), None)

    import ctypes
    bad_act = svdq.make_epilogue_next(7, None, None)
    half = svdq.make_epilogue_next(0, il, None)
    same = svdq.make_epilogue_next(1, il, word[0:])
    gelu = svdq.make_epilogue_next(1, None, None)
    assert fwd(w, None, ctypes.byref(bad_act)) == 1
    assert fwd(w, None, ctypes.byref(half)) == 1
    assert fwd(w, word.data_ptr(), ctypes.byref(same)) == 1  # next_amax is this call's x_amax
    assert fwd(w4, None, ctypes.byref(gelu)) == 1  # INT4 takes no epilogue extras
    unaligned = svdq.make_epilogue_next(1, il, word.data_ptr() + 2)
    assert fwd(w, None, ctypes.byref(unaligned)) == 3
    # the GEMM entry needs the amax for NVFP4
    qx = T.aligned_empty(M * 128)
    sx = T.aligned_empty(svdq.svdq_act_scale_bytes(w, M))
    assert lib.svdq_w4a4_gemm_lora_up_dyn(w.handle, qx.data_ptr(), sx.data_ptr(), None, None, M, None, None,
                                          Y.data_ptr(), 0, None) == 1
    assert lib.svdq_quantize_act_lora_down_dyn(w.handle, X.data_ptr(), M, None, qx.data_ptr(), sx.data_ptr(), None,
                                               None) == 1
    # a no-op epilogue is accepted for INT4, and the forward runs
    nop = svdq.make_epilogue_next(0, None, None)
    ws4 = _ws(svdq, w4, M)
    assert lib.svdq_linear_forward_dyn(w4.handle, X.data_ptr(), M, None, None, ctypes.byref(nop), Y.data_ptr(), 0,
                                       ws4.data_ptr(), ws4.numel(), None) == 0
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w4) == 0


@pytest.mark.parametrize("out_dtype", [0, 1], ids=["bf16", "f32"])
def test_dyn_qkv_prologue_equals_static(svdq, out_dtype):
    """The fused QKV projection with the dynamic scale (its own GEMM variant)
    gives the static projection's output bit for bit; the static one is
    checked against the oracle's prologue in the single-layer tests."""
    li = synth.make_layer("qkv", 31, M=300, K=512, N=768)
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M, N, heads = 300, 768, 2
    nq, nk, cs, sn = synth.qkv_prologue_inputs(M, 128, 23)
    dq, dk, dc, ds = T.dev_f32(nq), T.dev_f32(nk), T.dev_f32(cs.T.copy()), T.dev_f32(sn.T.copy())
    pro = svdq.make_qkv_prologue(heads, dq, dk, dc, ds, 1e-6)
    X = T.dev_u16(li.x_bits)
    ws = _ws(svdq, w, M)
    Yd = _ydev(M, N, out_dtype)
    svdq.svdq_linear_forward_dyn(w, X, M, None, Yd, ws, ws.numel(), pro=pro, out_dtype=out_dtype)
    Ys = _ydev(M, N, out_dtype)
    svdq.svdq_linear_forward_qkv(w, X, M, float(ol.gx), pro, Ys, ws, ws.numel(), out_dtype)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w) == 0
    assert torch.equal(Yd, Ys)


def test_dyn_forward_int4_ignores_the_scale_word(svdq):
    """INT4 has no tensor scale: the dynamic forward (with or without an amax
    word) is the static forward, bit for bit."""
    li = synth.make_layer("int4", 9, M=260, K=512, N=384)
    ol = T.oracle_layer(li, precision="int4")
    w = T.gpu_prepare(svdq, li, ol, "int4")
    M, N = 260, 384
    X = T.dev_u16(li.x_bits)
    ws = _ws(svdq, w, M)
    junk = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    Y0, Y1, Y2 = _ydev(M, N, 1), _ydev(M, N, 1), _ydev(M, N, 1)
    svdq.svdq_linear_forward(w, X, M, 1.0, Y0, ws, ws.numel(), 1)
    svdq.svdq_linear_forward_dyn(w, X, M, None, Y1, ws, ws.numel(), out_dtype=1)
    svdq.svdq_linear_forward_dyn(w, X, M, junk, Y2, ws, ws.numel(), out_dtype=1)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w) == 0
    assert torch.equal(Y0, Y1) and torch.equal(Y0, Y2)
