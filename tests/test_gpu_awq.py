"""Parity of the awq_w4a16 kernel family (through the C ABI) against the
CPU oracle: weight codes and scales bit-exact, Y within the fp32
accumulation bound (fp32 output) or that bound plus half a bf16 ulp (bf16
output), and within the layer bar of relative Frobenius error 2e-3."""
import numpy as np
import pytest
import torch

import synth
from oracle import awq as A
from tests import svdq_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def svdq():
    if not torch.cuda.is_available():
        pytest.fail("no CUDA device")
    from bit_diffusion_transformer_svdq_b200 import svdq as mod
    mod.load_library()
    return mod


def untile_gemv_codes(buf: np.ndarray, N: int, K: int) -> np.ndarray:
    """The GEMV tile layout of include/svdq.h back to N x K nibbles."""
    n = np.arange(N)[:, None]
    c = np.arange(K // 32)[None, :]
    base = ((n // 32) * (K // 32) + c) * 512 + (n % 32) * 16  # N x K/32: 16 bytes each
    idx = base[:, :, None] + np.arange(16)[None, None, :]
    packed = buf.reshape(-1)[idx].reshape(N, K // 2)
    return T.unpack_codes(packed)


def _prepare(svdq, li, alpha):
    W = T.dev_f32(li.w)
    a = T.dev_f32(alpha)
    b = T.dev_u16(li.bias_bits)
    return svdq.prepare_layer(W, a, None, None, b, 0, svdq.SVDQ_AWQ_W4A16)


def _check_y(y, ref, xh, prep, out_dtype):
    # fp32 accumulation bound: (K/64 + 72) roundings of magnitude sum |x s q|
    K = xh.shape[1]
    mag = np.abs(xh.astype(np.float64)) @ np.abs(A.Q.int4_dequantize(prep.q, prep.s)).T + np.abs(prep.bias)[None, :]
    bound = (K / 64 + 72) * 2.0 ** -24 * mag
    d = np.abs(y.astype(np.float64) - ref)
    if out_dtype == 0:
        bound = bound + 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
    assert np.all(d <= bound), float((d / np.maximum(bound, 1e-30)).max())
    assert np.linalg.norm(y - ref) / np.linalg.norm(ref) <= 2e-3


CASES = [
    ("m1_ragged_n", dict(M=1, K=192, N=80)),
    ("m3", dict(M=3, K=512, N=256)),
    ("m9_two_row_blocks", dict(M=9, K=1024, N=96)),
    ("m5", dict(M=5, K=256, N=512)),
    # long K: 24 groups per warp, so the rotating prefetch slots wrap many
    # times; four activation rows per CTA with a ragged last row block
    ("m1_long_k", dict(M=1, K=12288, N=128)),
    ("m4_long_k_ragged_n", dict(M=4, K=6144, N=208)),
]


@pytest.mark.parametrize("out_dtype", [1, 0], ids=["f32", "bf16"])
@pytest.mark.parametrize("name,over", CASES, ids=[c[0] for c in CASES])
def test_awq_parity(svdq, name, over, out_dtype):
    li = synth.make_layer("awq", 31, **over)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    alpha = synth.awq_alpha(K, 31)
    prep = A.prepare(li.w, alpha, li.bias)
    w = _prepare(svdq, li, alpha)
    v = w.view()  # qw is in the GEMV tile layout
    st = w.storage
    base = st.data_ptr()
    qbytes = st[v.qw - base: v.qw - base + v.n_pad * K // 2].cpu().numpy()
    codes = untile_gemv_codes(qbytes, N, K)
    assert np.array_equal(codes, (prep.q.astype(np.int16) & 0xF).astype(np.uint8))
    sw = st[v.sw - base: v.sw - base + v.sw_bytes].cpu().numpy().view(np.float16).reshape(K // 64, v.n_pad)
    assert np.array_equal(sw[:, :N].T.view(np.uint16), prep.s.view(np.uint16))
    assert np.all(sw[:, N:] == 0)

    X = T.dev_u16(li.x_bits)
    Y = torch.empty((M, N), dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
    svdq.svdq_awq_w4a16_forward(w, X, M, Y, out_dtype)
    assert svdq.svdq_device_status(w) == 0
    y = Y.float().cpu().numpy()
    ref = A.forward(li.x, prep)
    xh = (li.x * prep.inv_alpha[None, :]).astype(np.float32)
    _check_y(y, ref, xh, prep, out_dtype)


def test_awq_full_size_flux_modulation(svdq):
    """FLUX double-block adaLN modulation at full size: 3072 -> 18432, one
    row per image, batch of 1 and of 2."""
    li = synth.make_layer("awq", 5, M=2)
    M, K, N = li.shape.M, li.shape.K, li.shape.N
    alpha = synth.awq_alpha(K, 5)
    prep = A.prepare(li.w, alpha, li.bias)
    w = _prepare(svdq, li, alpha)
    X = T.dev_u16(li.x_bits)
    ref = A.forward(li.x, prep)
    xh = (li.x * prep.inv_alpha[None, :]).astype(np.float32)
    for rows in (1, 2):
        for out_dtype in (1, 0):
            Y = torch.empty((rows, N), dtype=torch.float32 if out_dtype == 1 else torch.bfloat16, device="cuda")
            svdq.svdq_awq_w4a16_forward(w, X, rows, Y, out_dtype)
            torch.cuda.synchronize()
            _check_y(Y.float().cpu().numpy(), ref[:rows], xh[:rows], prep, out_dtype)


def test_awq_argument_errors(svdq):
    lib = svdq.load_library()
    assert svdq.svdq_weights_bytes(svdq.LayerDesc(256, 64, 16, svdq.SVDQ_AWQ_W4A16, 64)) == 0  # rank must be 0
    assert svdq.svdq_weights_bytes(svdq.LayerDesc(256, 64, 0, svdq.SVDQ_AWQ_W4A16, 16)) == 0  # group 64
    li = synth.make_layer("awq", 3, M=2, K=128, N=64)
    w = _prepare(svdq, li, np.ones(128, np.float32))
    X = T.dev_u16(li.x_bits)
    Y = torch.empty((2, 64), dtype=torch.bfloat16, device="cuda")
    # the 4-bit-activation entry points refuse awq weights
    assert lib.svdq_quantize_act_lora_down(w.handle, X.data_ptr(), 2, 1.0, Y.data_ptr(), Y.data_ptr(), None, None) == 1
    assert lib.svdq_w4a4_gemm_lora_up(w.handle, X.data_ptr(), X.data_ptr(), 1.0, None, 2, Y.data_ptr(), 0, None) == 1
    # and the awq entry refuses 4-bit-activation weights
    li2 = synth.make_layer("tiny", 3)
    ol = T.oracle_layer(li2)
    w2 = T.gpu_prepare(svdq, li2, ol)
    assert lib.svdq_awq_w4a16_forward(w2.handle, X.data_ptr(), 2, Y.data_ptr(), 0, None) == 1
    assert lib.svdq_awq_w4a16_forward(w.handle, X.data_ptr() + 2, 2, Y.data_ptr(), 0, None) == 3
    assert lib.svdq_awq_w4a16_forward(w.handle, X.data_ptr(), -1, Y.data_ptr(), 0, None) == 2
    assert lib.svdq_awq_w4a16_forward(w.handle, X.data_ptr(), 0, Y.data_ptr(), 0, None) == 0
