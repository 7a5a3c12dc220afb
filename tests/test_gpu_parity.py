"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Bit-exact: lambda, inv_lambda, g_w, g_x, weight codes and scales, L1s,
activation codes and scales.  Tolerance (fp32 output mode): relative
Frobenius error <= 2e-3 and max |error| <= 1e-2 * rms(Y*) against the
oracle's fp64 Y* computed from the same codes.  bf16 output mode: the same
relative Frobenius bound, and per element |Y - Y*| <= 1e-2 rms(Y*) plus half
a bf16 ulp of Y* (the output rounding itself).
"""
import numpy as np
import pytest
import torch

import synth
from oracle import formats as F
from oracle import quant as Q
from oracle import svdq as V
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu

REL_F = 2e-3
MAX_ABS = 1e-2


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def test_device_is_supported(svdq):
    assert svdq.svdq_check_device(torch.cuda.current_device()) == 0


# (name, workload, overrides) -- reduced cases keep the distributions and
# span several tiles with ragged tails
CASES = [
    ("tiny", "tiny", {}),
    ("qkv_ragged", "qkv", dict(M=300, K=1024, N=768)),
    ("partial_k_n_rank64", "mlp_up", dict(M=129, K=320, N=144, rank=64)),
    ("rank0", "stack_out", dict(M=200, K=512, N=512, rank=0)),
    ("rank8", "mlp_down", dict(M=77, K=768, N=272, rank=8)),
    # more output tiles than CTAs: the persistent GEMMs wrap around the tile list
    ("many_tiles", "qkv", dict(M=2048, K=320, N=2560)),
]


def _layer(workload, over, seed=11):
    return synth.make_layer(workload, seed, **over)


def test_smoothing_lambda_bit_exact(svdq):
    for wl, over in [("tiny", {}), ("qkv", dict(M=300, K=1024, N=768))]:
        li = _layer(wl, over)
        X = T.dev_u16(li.x_bits)
        W = T.dev_f32(li.w)
        K = li.shape.K
        lam = torch.empty(K, dtype=torch.float32, device="cuda")
        scratch = torch.empty(2 * K, dtype=torch.float32, device="cuda")
        svdq.svdq_smoothing_lambda(X, W, lam, scratch)
        got = lam.cpu().numpy()
        ref = V.smoothing_lambda(li.x, li.w)
        assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


@pytest.mark.parametrize("precision", ["nvfp4", "int4"])
@pytest.mark.parametrize("name,wl,over", CASES, ids=[c[0] for c in CASES])
def test_prepare_weights_bit_exact(svdq, name, wl, over, precision):
    li = _layer(wl, over)
    ol = T.oracle_layer(li, precision=precision)
    w = T.gpu_prepare(svdq, li, ol, precision)
    torch.cuda.synchronize()
    h = T.weights_to_host(w)
    N, K = li.shape.N, li.shape.K
    p = ol.prep
    assert h["g_w"] == p.g_w
    assert np.array_equal(h["inv"].view(np.uint32), p.inv_lam.view(np.uint32))
    assert np.array_equal(T.unpack_codes(h["qw"]), p.qw if precision == "nvfp4" else (p.qw.astype(np.int16) & 0xF).astype(np.uint8))
    if precision == "nvfp4":
        assert np.array_equal(T.untile_nvfp4_scales(h["sw"], N, K), p.sw)
    else:
        sw = h["sw"].view(np.float16).reshape(K // 64, h["n_pad"])[:, :N].T
        assert np.array_equal(sw.view(np.uint16), p.sw.view(np.uint16))
    r = p.rank
    assert np.array_equal(h["l1s"][:r], T.bf16_bits(p.L1s))
    assert np.all(h["l1s"][r:] == 0)
    assert np.array_equal(h["l2"][:, :r], p.L2) and np.all(h["l2"][:, r:] == 0)
    assert np.array_equal(h["bias"], li.bias)


def test_act_global_scale_bit_exact(svdq):
    li = _layer("qkv", dict(M=300, K=1024, N=768))
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    g = torch.empty(1, dtype=torch.float32, device="cuda")
    svdq.svdq_act_global_scale(w, T.dev_u16(li.x_bits), g)
    assert g.item() == ol.gx


def _check_act_codes(svdq, w, li, ol, qx, sx, la, precision):
    M, K = li.shape.M, li.shape.K
    act = V.quantize_activations(li.x, ol.prep, ol.gx)
    got_codes = T.unpack_codes(qx[:M * K // 2].cpu().numpy().reshape(M, K // 2))
    if precision == "nvfp4":
        assert np.array_equal(got_codes, act.qx)
        sxh = sx.cpu().numpy()
        assert np.array_equal(T.untile_nvfp4_scales(sxh, M, K), act.sx)
        mp = (M + 127) // 128 * 128
        pad = T.tiled_scale_index(mp, K)[M:]
        assert np.all(sxh[pad] == 0)
    else:
        assert np.array_equal(T.nibbles_to_int(got_codes), act.qx)
        # the E4M3 copy of the codes the GEMM reads, after the packed codes
        nb = svdq.svdq_act_codes_bytes(w, M)
        assert np.array_equal(qx[nb - M * K:nb].cpu().numpy().reshape(M, K), T.e4m3_bytes(act.qx))
        mp = (M + 127) // 128 * 128
        sxh = sx.cpu().numpy().view(np.float16).reshape(K // 64, mp)
        assert np.array_equal(sxh[:, :M].T.view(np.uint16), act.sx.view(np.uint16))
    if la is not None:
        gw = ol.prep.g_w
        scale = np.float32(1.0) / np.float32(np.float32(ol.gx) * gw) if precision == "nvfp4" else np.float32(1.0)
        ref = act.lora_act * float(scale)
        got = la.cpu().numpy()[:, :ol.prep.rank].astype(np.float64)
        mag = (np.abs(li.x).astype(np.float64) @ np.abs(ol.prep.L1s).astype(np.float64).T) * float(scale)
        assert np.all(np.abs(got - ref) <= 2.0 ** -11 * np.abs(ref) + 1e-5 * mag + 1e-30)
        assert np.all(la.cpu().numpy()[:, ol.prep.rank:] == 0)
    return act


@pytest.mark.parametrize("precision", ["nvfp4", "int4"])
@pytest.mark.parametrize("name,wl,over", CASES, ids=[c[0] for c in CASES])
def test_quantize_act_lora_down_bit_exact(svdq, name, wl, over, precision):
    li = _layer(wl, over)
    ol = T.oracle_layer(li, precision=precision)
    w = T.gpu_prepare(svdq, li, ol, precision)
    X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
    _check_act_codes(svdq, w, li, ol, qx, sx, la, precision)


def test_quantize_rounding_ties_and_signed_zero(svdq):
    """Inputs built so that lambda = 1, g_x = 1 and every group's amax is 6 *
    (an E4M3 value or an E4M3 rounding tie): the E2M1 element ties
    (0.25, 0.75, ... , 5), negative values that round to -0, and the scale
    ties (incl. the subnormal ones) all reach the hardware conversions."""
    K, N = 256, 256
    e4m3_vals = F.e4m3_decode(np.arange(1, 0x7F, dtype=np.uint8))
    ties = (e4m3_vals[:-1] + e4m3_vals[1:]) / 2
    sub_ties = np.array([2 ** -10, 3 * 2 ** -10, 5 * 2 ** -10, 7 * 2 ** -10])
    t_all = np.concatenate([e4m3_vals, ties, sub_ties])
    t_all = t_all[t_all * 6 < 2 ** 15]
    body = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -0.125, -2.5, -5.0, 0.0, 1.0, -6.0, 4.0], np.float64)
    rows = []
    for i in range(0, len(t_all), K // 16):
        chunk = t_all[i:i + K // 16]
        r = np.zeros(K)
        for j, t in enumerate(chunk):
            g = np.concatenate([[6.0], body]) * t
            r[16 * j:16 * j + 16] = g
        rows.append(r)
    x = np.array(rows, np.float32)
    M = x.shape[0]
    assert np.array_equal(F.bf16_rn(x), x.astype(np.float64))  # bf16-exact inputs
    x_bits = T.bf16_bits(x)
    lam = np.ones(K, np.float32)
    rng = np.random.default_rng(3)
    w = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    li = synth.LayerInputs(synth.WORKLOADS["tiny"], 0, x_bits, x, w, T.bf16_bits(np.zeros(N)), np.zeros(N, np.float32))
    ol = T.oracle_layer(li, rank=0, lam=lam)
    gx = np.float32(1.0)
    ol.gx = gx
    w_gpu = T.gpu_prepare(svdq, li, ol)
    X, qx, sx, la = T.gpu_quantize(svdq, w_gpu, x_bits, 1.0)
    act = V.quantize_activations(x, ol.prep, gx)
    assert np.any(act.qx == 8)  # -0 codes are present
    got = T.unpack_codes(qx[:M * K // 2].cpu().numpy().reshape(M, K // 2))
    assert np.array_equal(got, act.qx)
    assert np.array_equal(T.untile_nvfp4_scales(sx.cpu().numpy(), M, K), act.sx)


def _forward_case(svdq, li, ol, precision, out_dtype):
    w = T.gpu_prepare(svdq, li, ol, precision)
    M, N = li.shape.M, li.shape.N
    X = T.dev_u16(li.x_bits)
    ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
    Y = torch.empty((M, N), dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    svdq.svdq_linear_forward(w, X, M, float(ol.gx), Y, ws, ws.numel(), out_dtype)
    assert svdq.svdq_device_status(w) == 0
    return w, Y.float().cpu().numpy()


def _assert_y(y, ref, out_dtype):
    st = T.y_error_stats(y, ref)
    assert st["rel_f"] <= REL_F, st
    rms = np.sqrt(np.mean(ref ** 2))
    if out_dtype == 1:
        assert st["max_abs_over_rms"] <= MAX_ABS, st
    else:
        half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
        assert np.all(np.abs(y - ref) <= MAX_ABS * rms + half_ulp), st


@pytest.mark.parametrize("out_dtype", [1, 0], ids=["f32", "bf16"])
@pytest.mark.parametrize("name,wl,over", CASES, ids=[c[0] for c in CASES])
def test_forward_parity_nvfp4(svdq, name, wl, over, out_dtype):
    li = _layer(wl, over)
    ol = T.oracle_layer(li, precision="nvfp4")
    w, y = _forward_case(svdq, li, ol, "nvfp4", out_dtype)
    ref = V.forward(li.x, ol.prep, ol.gx)
    _assert_y(y, ref, out_dtype)


def test_gemm_exact_on_integer_grid(svdq):
    """With lambda = 1, rank 0, power-of-two scales and g_x = g_w = 1 the
    4-bit product is a sum of short binary fractions that fp32 holds
    exactly: the tensor-core result must equal the oracle bit for bit.
    This pins the code nibble order, the K order and the scale layouts."""
    rng = np.random.default_rng(5)
    M, K, N = 192, 512, 384
    grid = np.concatenate([F.E2M1_GRID, -F.E2M1_GRID])
    pow2 = np.array([0.5, 1.0, 2.0])
    # weights: each group holds a 6 (so amax = 6 s) times a power-of-two scale s
    e_w = rng.choice(grid, size=(N, K))
    e_w[:, ::16] = 6.0
    s_w = rng.choice(pow2, size=(N, K // 16))
    W = e_w * np.repeat(s_w, 16, axis=1)
    W[0, 0] = 6.0 * 448.0  # amax = 2688 makes g_w = 1 (that group's scale is 448)
    W[0, 1:16] = 0.0
    W = W.astype(np.float32)
    li = synth.LayerInputs(synth.WORKLOADS["tiny"], 0, np.zeros((M, K), np.uint16), np.zeros((M, K), np.float32), W,
                           T.bf16_bits(np.zeros(N)), np.zeros(N, np.float32))
    ol = T.oracle_layer(li, rank=0, lam=np.ones(K, np.float32))
    assert ol.prep.g_w == 1.0
    w = T.gpu_prepare(svdq, li, ol)
    # activations: random codes and power-of-two scales given directly to the GEMM
    codes = rng.integers(0, 16, size=(M, K)).astype(np.uint8)
    sx_codes = F.e4m3_encode(rng.choice(pow2, size=(M, K // 16)))
    qx = torch.from_numpy(F.pack_nibbles(codes)).cuda()
    mp = (M + 127) // 128 * 128
    sx = torch.from_numpy(T.tile_nvfp4_scales(sx_codes, mp, K)).cuda()
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    svdq.svdq_w4a4_gemm_lora_up(w, qx, sx, 1.0, None, M, Y, 1)
    torch.cuda.synchronize()
    act = V.ActQuant(codes, sx_codes, np.zeros((M, 0)))
    ref = V.forward_from_codes(act, ol.prep, np.float32(1.0))
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), ref)


@pytest.mark.parametrize("out_dtype", [1, 0], ids=["f32", "bf16"])
@pytest.mark.parametrize("name,wl,over", CASES, ids=[c[0] for c in CASES])
def test_forward_parity_int4(svdq, name, wl, over, out_dtype):
    li = _layer(wl, over)
    ol = T.oracle_layer(li, precision="int4")
    w, y = _forward_case(svdq, li, ol, "int4", out_dtype)
    ref = V.forward(li.x, ol.prep)
    _assert_y(y, ref, out_dtype)


def test_int4_gemm_exact_on_integer_grid(svdq):
    """INT4 counterpart of the exactness pin: lambda = 1, rank 0, integer
    codes and power-of-two fp16 scales make every partial sum an fp32-exact
    value, so the kind::f8f6f4 product of the E4M3 codes with its per-group
    scaling must equal the oracle bit for bit.  This pins the E4M3 copies of
    both operands (the activations' written here from the definition, after
    the packed codes in the same buffer) and both scale layouts.
    K = 576 is an odd number of 64-groups (a half-filled last ring stage)."""
    rng = np.random.default_rng(9)
    M, K, N = 200, 576, 320
    pow2 = np.array([0.25, 0.5, 1.0, 2.0])
    # weights: every 64-group holds a 7 (amax = 7 s) so that the codes are W / s exactly
    q_w = rng.integers(-7, 8, size=(N, K))
    q_w[:, ::64] = 7
    s_w = rng.choice(pow2, size=(N, K // 64))
    W = (q_w * np.repeat(s_w, 64, axis=1)).astype(np.float32)
    li = synth.LayerInputs(synth.WORKLOADS["tiny"], 0, np.zeros((M, K), np.uint16), np.zeros((M, K), np.float32), W,
                           T.bf16_bits(np.zeros(N)), np.zeros(N, np.float32))
    ol = T.oracle_layer(li, precision="int4", rank=0, lam=np.ones(K, np.float32))
    assert np.array_equal(ol.prep.qw.astype(np.int64), q_w)
    w = T.gpu_prepare(svdq, li, ol, "int4")
    codes = rng.integers(-8, 8, size=(M, K)).astype(np.int8)
    sx = rng.choice(pow2, size=(M, K // 64)).astype(np.float16)
    mp = (M + 127) // 128 * 128
    sx_dev = np.zeros((K // 64, mp), np.float16)
    sx_dev[:, :M] = sx.T
    nb = svdq.svdq_act_codes_bytes(w, M)
    buf = np.zeros(nb, np.uint8)
    buf[:M * K // 2] = F.pack_nibbles((codes.astype(np.int16) & 0xF).astype(np.uint8)).ravel()
    buf[nb - M * K:] = T.e4m3_bytes(codes).ravel()
    qx = torch.from_numpy(buf).cuda()
    sxt = torch.from_numpy(sx_dev.view(np.uint16).astype(np.int16)).cuda()
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    svdq.svdq_w4a4_gemm_lora_up(w, qx, sxt, 1.0, None, M, Y, 1)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w) == 0
    act = V.ActQuant(codes, sx, np.zeros((M, 0)))
    ref = V.forward_from_codes(act, ol.prep)
    assert np.array_equal(Y.cpu().numpy().astype(np.float64), ref)


def _rn32(fr):
    """fp32 round-to-nearest-even of an exact rational (normal range)."""
    from fractions import Fraction
    if fr == 0:
        return np.float32(0.0)
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    scale = Fraction(2) ** (23 - e)  # a * scale in [2^23, 2^24)
    x = a * scale
    n = x.numerator // x.denominator
    rem = x - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    v = np.float32(float(Fraction(n) / scale))
    return -v if fr < 0 else v


def test_int4_gemm_rounds_once_per_group(svdq):
    """The INT4 GEMM's accumulation with arbitrary fp16 scales: for every
    output, acc = RN32(P_g s_w s_x + acc) group after group (P_g the exact
    integer group sum), one rounding per group, then + b (0 here).  The
    expected values are exact rationals rounded to fp32 here, so fp32 Y
    must match bit for bit.  Rank 0, lambda = 1, four groups."""
    from fractions import Fraction
    rng = np.random.default_rng(21)
    M, K, N = 64, 256, 128
    G = K // 64
    s_w = (rng.uniform(0.5, 2.0, size=(N, G)) * 2.0 ** rng.integers(-6, 2, size=(N, G))).astype(np.float16)
    q_w = rng.integers(-7, 8, size=(N, K))
    q_w[:, ::64] = 7  # every group's amax is 7 s_w: the codes are W / s_w exactly
    W = (q_w * np.repeat(s_w.astype(np.float32), 64, axis=1)).astype(np.float32)
    li = synth.LayerInputs(synth.WORKLOADS["tiny"], 0, np.zeros((M, K), np.uint16), np.zeros((M, K), np.float32), W,
                           T.bf16_bits(np.zeros(N)), np.zeros(N, np.float32))
    ol = T.oracle_layer(li, precision="int4", rank=0, lam=np.ones(K, np.float32))
    assert np.array_equal(ol.prep.qw.astype(np.int64), q_w)
    assert np.array_equal(ol.prep.sw.view(np.uint16), s_w.view(np.uint16))
    w = T.gpu_prepare(svdq, li, ol, "int4")
    codes = rng.integers(-8, 8, size=(M, K)).astype(np.int8)
    sx = (rng.uniform(0.5, 2.0, size=(M, G)) * 2.0 ** rng.integers(-6, 2, size=(M, G))).astype(np.float16)
    mp = (M + 127) // 128 * 128
    sx_dev = np.zeros((G, mp), np.float16)
    sx_dev[:, :M] = sx.T
    nb = svdq.svdq_act_codes_bytes(w, M)
    buf = np.zeros(nb, np.uint8)
    buf[:M * K // 2] = F.pack_nibbles((codes.astype(np.int16) & 0xF).astype(np.uint8)).ravel()
    buf[nb - M * K:] = T.e4m3_bytes(codes).ravel()
    Y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    svdq.svdq_w4a4_gemm_lora_up(w, torch.from_numpy(buf).cuda(),
                                torch.from_numpy(sx_dev.view(np.uint16).astype(np.int16)).cuda(), 1.0, None, M, Y, 1)
    torch.cuda.synchronize()
    assert svdq.svdq_device_status(w) == 0
    y = Y.cpu().numpy()
    P = np.einsum("mgk,ngk->mng", codes.astype(np.int64).reshape(M, G, 64), q_w.reshape(N, G, 64))
    fw = [[Fraction(float(v)) for v in row] for row in s_w.astype(np.float64)]
    fx = [[Fraction(float(v)) for v in row] for row in sx.astype(np.float64)]
    for m in range(M):
        for n in range(N):
            acc = np.float32(0.0)
            for g in range(G):
                acc = _rn32(int(P[m, n, g]) * fw[n][g] * fx[m][g] + Fraction(float(acc)))
            assert y[m, n].view(np.uint32) == acc.view(np.uint32), (m, n, y[m, n], acc)


def test_argument_errors(svdq):
    li = _layer("tiny", {})
    ol = T.oracle_layer(li)
    w = T.gpu_prepare(svdq, li, ol)
    M = li.shape.M
    X = T.dev_u16(li.x_bits)
    ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
    Y = torch.empty((M, li.shape.N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(svdq.SVDQError) as e:
        svdq.svdq_linear_forward(w, X, M, float(ol.gx), Y, ws, ws.numel() - 1024)
    assert e.value.status == 7
    with pytest.raises(svdq.SVDQError) as e:
        svdq.svdq_linear_forward(w, X, M, 0.0, Y, ws, ws.numel())
    assert e.value.status == 1
    with pytest.raises(svdq.SVDQError) as e:
        svdq.svdq_linear_forward(w, X, M, float(ol.gx), Y.reshape(-1).view(torch.uint8)[2:], ws, ws.numel())
    assert e.value.status == 3
    svdq.svdq_linear_forward(w, X, 0, float(ol.gx), Y, ws, ws.numel())  # M = 0 is a no-op
    bad = svdq.make_desc(100, 256, 16)
    assert svdq.svdq_weights_bytes(bad) == 0


# ------------------------------------------------ fused QKV attention prologue
# (heads, workload, overrides): N = 3 * heads * 128; ragged M, several tiles
QKV_CASES = [
    ("h2_ragged", 2, "qkv", dict(M=300, K=512, N=768)),
    ("h4_rank16", 4, "qkv", dict(M=129, K=256, N=1536, rank=16)),
    ("h2_rank0", 2, "stack_qkv", dict(M=64, K=320, N=768, rank=0)),
]


def _qkv_case(svdq, li, ol, heads, precision, out_dtype, through_forward=True):
    from oracle import qkv as A
    w = T.gpu_prepare(svdq, li, ol, precision)
    M, N = li.shape.M, li.shape.N
    nq, nk, cs, sn = synth.qkv_prologue_inputs(M, 128, 23)
    # the library takes the tables frequency-major (head_dim/2 x M)
    dq, dk, dc, ds = T.dev_f32(nq), T.dev_f32(nk), T.dev_f32(cs.T.copy()), T.dev_f32(sn.T.copy())
    eps = 1e-6
    pro = svdq.make_qkv_prologue(heads, dq, dk, dc, ds, eps)
    X = T.dev_u16(li.x_bits)
    Y = torch.empty((M, N), dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    gx = float(ol.gx)
    if through_forward:
        ws = T.aligned_empty(svdq.svdq_workspace_bytes(w, M))
        svdq.svdq_linear_forward_qkv(w, X, M, gx, pro, Y, ws, ws.numel(), out_dtype)
    else:
        _, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, gx)
        svdq.svdq_w4a4_gemm_lora_up_qkv(w, qx, sx, gx, la, M, pro, Y, out_dtype)
    assert svdq.svdq_device_status(w) == 0
    y = Y.float().cpu().numpy()
    plain = V.forward(li.x, ol.prep, ol.gx if precision == "nvfp4" else None)
    ref = A.qkv_prologue(plain, heads, 128, nq, nk, cs, sn, eps)
    return y, ref


@pytest.mark.parametrize("precision", ["nvfp4", "int4"])
@pytest.mark.parametrize("out_dtype", [1, 0], ids=["f32", "bf16"])
@pytest.mark.parametrize("name,heads,wl,over", QKV_CASES, ids=[c[0] for c in QKV_CASES])
def test_qkv_prologue_parity(svdq, name, heads, wl, over, out_dtype, precision):
    li = _layer(wl, over)
    ol = T.oracle_layer(li, precision=precision)
    y, ref = _qkv_case(svdq, li, ol, heads, precision, out_dtype, through_forward=(name != "h4_rank16"))
    w = heads * 128
    for sec in range(3):  # Q, K (normalised, unit scale) and V (the layer's own scale) separately
        _assert_y(y[:, sec * w:(sec + 1) * w], ref[:, sec * w:(sec + 1) * w], out_dtype)


def test_qkv_prologue_argument_errors(svdq):
    li = _layer("qkv", dict(M=64, K=256, N=768))
    ol = T.oracle_layer(li, precision="nvfp4")
    w = T.gpu_prepare(svdq, li, ol, "nvfp4")
    M = 64
    X, qx, sx, la = T.gpu_quantize(svdq, w, li.x_bits, float(ol.gx))
    t = torch.ones(M * 64 + 4, dtype=torch.float32, device="cuda")
    Y = torch.empty((M, 768), dtype=torch.bfloat16, device="cuda")
    lib = svdq.load_library()
    import ctypes

    def call(pro):
        return lib.svdq_w4a4_gemm_lora_up_qkv(w.handle, qx.data_ptr(), sx.data_ptr(), float(ol.gx), la.data_ptr(), M,
                                              ctypes.byref(pro), Y.data_ptr(), 0, None)

    good = svdq.make_qkv_prologue(2, t, t, t, t, 1e-6)
    assert call(good) == 0
    torch.cuda.synchronize()
    assert call(svdq.make_qkv_prologue(3, t, t, t, t, 1e-6)) == 2          # N != 3 * heads * 128 (and odd)
    assert call(svdq.make_qkv_prologue(2, t, t, t, t, 1e-6, head_dim=64)) == 2
    assert call(svdq.make_qkv_prologue(2, t, t, t, t, 0.0)) == 1          # eps must be > 0
    assert call(svdq.make_qkv_prologue(2, None, t, t, t, 1e-6)) == 1
    assert call(svdq.make_qkv_prologue(2, t, t, t[1:], t, 1e-6)) == 3     # rope_cos not 16-byte aligned
