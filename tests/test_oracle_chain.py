"""Pins of the oracle's chained-layer pieces (no GPU): the tanh-form GELU
against a library routine, its odd-part identity and the erf form it
approximates; the next layer's amax against a brute-force loop; and the
dynamic tensor scale of a chain against the calibration formula."""
import math

import numpy as np
import scipy.special
import torch

import synth
from oracle import chain as C
from oracle import formats as F
from oracle import quant as Q
from oracle import svdq as V

GRID = np.concatenate([np.linspace(-12.0, 12.0, 4801), [-1e3, -40.0, 0.0, 1e-30, 40.0, 1e3]])


def test_gelu_tanh_matches_torch_tanh_approximation():
    ref = torch.nn.functional.gelu(torch.from_numpy(GRID), approximate="tanh").numpy()
    got = C.gelu_tanh(GRID)
    # same formula, other evaluation order: agreement to fp64 rounding
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_gelu_tanh_odd_part_is_identity():
    # tanh is odd, so gelu(y) - gelu(-y) = 0.5 y (1 + t) + 0.5 y (1 - t) = y
    y = GRID[np.abs(GRID) < 50]
    assert np.allclose(C.gelu_tanh(y) - C.gelu_tanh(-y), y, rtol=1e-14, atol=1e-14)


def test_gelu_tanh_special_values():
    assert C.gelu_tanh(0.0) == 0.0
    assert C.gelu_tanh(1e3) == 1e3  # tanh saturates at 1
    assert C.gelu_tanh(-1e3) == 0.0 or abs(C.gelu_tanh(-1e3)) < 1e-300
    # at y = 1: u = sqrt(2/pi) * 1.044715
    u = math.sqrt(2.0 / math.pi) * 1.044715
    assert math.isclose(float(C.gelu_tanh(1.0)), 0.5 * (1.0 + math.tanh(u)), rel_tol=1e-15)


def test_gelu_tanh_close_to_erf_gelu():
    # the tanh form approximates 0.5 y (1 + erf(y / sqrt 2)) to within 5e-4
    exact = 0.5 * GRID * (1.0 + scipy.special.erf(GRID / math.sqrt(2.0)))
    assert np.max(np.abs(C.gelu_tanh(GRID) - exact)) < 5e-4


def test_gelu_tanh_equals_sigmoid_form():
    # 0.5 (1 + tanh(u)) = 1 / (1 + exp(-2u)); the tanh form loses the far
    # negative tail to cancellation in 1 + tanh (absolute error ~1e-16 |y|)
    y = GRID[np.abs(GRID) < 30]
    u = C.GELU_K0 * (y + C.GELU_K1 * y ** 3)
    assert np.allclose(C.gelu_tanh(y), y / (1.0 + np.exp(-2.0 * u)), rtol=1e-12, atol=1e-14)


def F_bf16(a):
    return F.bf16_rn(a).astype(np.float32)


def test_act_amax_brute_force():
    rng = np.random.default_rng(3)
    x = F_bf16(rng.normal(size=(5, 32)) * 3.0)
    il = (rng.uniform(0.25, 4.0, size=32)).astype(np.float32)
    best = np.float32(0.0)
    for m in range(5):
        for k in range(32):
            v = abs(np.float32(np.float32(x[m, k]) * il[k]))
            if v > best:
                best = v
    assert C.act_amax(x, il) == best
    assert C.act_amax(np.zeros((0, 32), np.float32), il) == 0.0


def test_round_output_bf16_is_representable_and_nearest():
    rng = np.random.default_rng(4)
    y = rng.normal(size=1000) * 10.0
    r = C.round_output(y, "bf16").astype(np.float64)
    bits = r.astype(np.float32).view(np.uint32)
    assert np.all(bits & 0xFFFF == 0)  # bf16 values
    ulp = 2.0 ** (np.floor(np.log2(np.abs(y))) - 7)
    assert np.all(np.abs(r - y) <= ulp / 2)


def test_chain_scale_matches_calibration_formula():
    li_a = synth.make_layer("mlp_up", 5, M=40, K=128, N=96)
    li_b = synth.make_layer("mlp_down", 6, M=40, K=96, N=64)
    lam_a = V.smoothing_lambda(li_a.x, li_a.w)
    lam_b = V.smoothing_lambda(li_b.x, li_b.w)
    pa = V.prepare_weights(li_a.w, lam_a, *V.lowrank_factors(li_a.w, lam_a, 8), li_a.bias)
    pb = V.prepare_weights(li_b.w, lam_b, *V.lowrank_factors(li_b.w, lam_b, 8), li_b.bias)
    ya, amax_b, yb = C.chain_forward(li_a.x, pa, pb)
    # the stored output is the rounded GELU of layer a's forward
    ref_a = C.gelu_tanh(V.forward(li_a.x, pa, V.act_global_scale(li_a.x, pa.inv_lam)))
    assert np.array_equal(ya, C.round_output(ref_a, "bf16"))
    # the next amax is the calibration amax of that output
    assert Q.nvfp4_tensor_scale(amax_b) == V.act_global_scale(ya, pb.inv_lam)
    # GELU output is bounded below by its minimum, about -0.17
    assert ya.min() > -0.2
    assert yb.shape == (40, 64) and np.all(np.isfinite(yb))


def test_dynamic_scale_is_the_default():
    li = synth.make_layer("mlp_up", 8, M=33, K=128, N=64)
    lam = V.smoothing_lambda(li.x, li.w)
    p = V.prepare_weights(li.w, lam, *V.lowrank_factors(li.w, lam, 8), li.bias)
    g = V.act_global_scale(li.x, p.inv_lam)
    a0, a1 = V.quantize_activations(li.x, p, None), V.quantize_activations(li.x, p, g)
    assert np.array_equal(a0.qx, a1.qx) and np.array_equal(a0.sx, a1.sx)
    assert np.any(a0.qx != 0)
    assert np.array_equal(V.forward(li.x, p), V.forward(li.x, p, g))
    # a different scale gives different scale codes
    a2 = V.quantize_activations(li.x, p, np.float32(g * 2))
    assert not np.array_equal(a2.sx, a1.sx)
