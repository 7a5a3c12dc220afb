"""Helpers shared by the GPU parity tests: uploading the seeded inputs,
running the CUDA path through the C ABI, running the oracle on the same
inputs, and the scale-layout index map documented in include/svdq.h."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import synth
from oracle import formats as F
from oracle import svdq as V

PREC = {"nvfp4": 0, "int4": 1}


def tiled_scale_index(rows: int, K: int) -> np.ndarray:
    """Flat byte offset of (row m, 16-group j) in the tiled NVFP4 scale
    layout of include/svdq.h, as an array of shape (rows, K/16)."""
    m = np.arange(rows)[:, None]
    j = np.arange(K // 16)[None, :]
    return ((m // 128) * (K // 64) + j // 4) * 512 + (m % 32) * 16 + ((m // 32) % 4) * 4 + j % 4


def untile_nvfp4_scales(buf: np.ndarray, rows: int, K: int) -> np.ndarray:
    return buf.reshape(-1)[tiled_scale_index(rows, K)]


def tile_nvfp4_scales(canon: np.ndarray, rows_padded: int, K: int) -> np.ndarray:
    out = np.zeros(rows_padded * K // 16, np.uint8)
    out[tiled_scale_index(canon.shape[0], K)] = canon
    return out


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def nibbles_to_int(n: np.ndarray) -> np.ndarray:
    n = n.astype(np.int16)
    return np.where(n >= 8, n - 16, n).astype(np.int8)


def aligned_empty(nbytes: int, device="cuda") -> torch.Tensor:
    buf = torch.empty(nbytes + 1024, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 1024
    return buf[off:off + nbytes]


def dev_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def bf16_bits(a: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_from_f32(np.asarray(a, np.float32))


@dataclasses.dataclass
class OracleLayer:
    lam: np.ndarray
    L1: np.ndarray
    L2: np.ndarray
    prep: V.Prepared
    gx: np.float32


def oracle_layer(li: synth.LayerInputs, rank: int | None = None, precision: str | None = None,
                 lam: np.ndarray | None = None) -> OracleLayer:
    rank = li.shape.rank if rank is None else rank
    precision = li.shape.precision if precision is None else precision
    if lam is None:
        lam = V.smoothing_lambda(li.x, li.w)
    L1, L2 = V.lowrank_factors(li.w, lam, rank)
    prep = V.prepare_weights(li.w, lam, L1, L2, li.bias, precision)
    gx = V.act_global_scale(li.x, prep.inv_lam) if precision == "nvfp4" else np.float32(1.0)
    return OracleLayer(lam, L1, L2, prep, gx)


def gpu_prepare(svdq, li: synth.LayerInputs, ol: OracleLayer, precision: str | None = None):
    precision = li.shape.precision if precision is None else precision
    rank = ol.L1.shape[0]
    W = dev_f32(li.w)
    lam = dev_f32(ol.lam)
    L1 = dev_u16(bf16_bits(ol.L1)) if rank else None
    L2 = dev_u16(bf16_bits(ol.L2)) if rank else None
    b = dev_u16(li.bias_bits)
    w = svdq.prepare_layer(W, lam, L1, L2, b, rank, PREC[precision])
    return w


def gpu_quantize(svdq, w, x_bits: np.ndarray, gx: float):
    M, K = x_bits.shape
    X = dev_u16(x_bits)
    qx = aligned_empty(max(svdq.svdq_act_codes_bytes(w, M), 16))
    sx = aligned_empty(max(svdq.svdq_act_scale_bytes(w, M), 16))
    rp = w.view().rank_pad
    la = torch.empty((M, rp), dtype=torch.float32, device="cuda") if rp else None
    svdq.svdq_quantize_act_lora_down(w, X, M, gx, qx, sx, la)
    torch.cuda.synchronize()
    return X, qx, sx, la


def weights_to_host(w):
    v = w.view()
    K, N, rp = v.K, v.N, v.rank_pad
    st = w.storage
    base = st.data_ptr()

    def grab(ptr, nbytes):
        off = ptr - base
        return st[off:off + nbytes].cpu().numpy()

    qw = grab(v.qw, N * K // 2).reshape(N, K // 2)
    sw = grab(v.sw, v.sw_bytes)
    l1s = grab(v.l1s, rp * K * 2).view(np.uint16).reshape(rp, K) if rp else np.zeros((0, K), np.uint16)
    l2 = grab(v.l2, N * rp * 4).view(np.float32).reshape(N, rp) if rp else np.zeros((N, 0), np.float32)
    inv = grab(v.inv_lambda, K * 4).view(np.float32)
    bias = grab(v.bias, N * 4).view(np.float32)
    return dict(qw=qw, sw=sw, l1s=l1s, l2=l2, inv=inv, bias=bias, g_w=np.float32(v.g_w), n_pad=v.n_pad, rank_pad=rp)


def y_error_stats(y: np.ndarray, ref: np.ndarray) -> dict:
    d = y.astype(np.float64) - ref
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return dict(rel_f=float(np.linalg.norm(d) / np.linalg.norm(ref)), max_abs_over_rms=float(np.abs(d).max() / rms))


def expected_weights(li: synth.LayerInputs, prep: V.Prepared) -> dict:
    """The oracle's prepared weights in the canonical layout that
    svdq_export_weights writes (codes packed two per byte, even k low)."""
    qw = prep.qw if prep.precision == "nvfp4" else F.int4_to_nibble(prep.qw)
    sw = prep.sw if prep.precision == "nvfp4" else prep.sw.view(np.uint16)
    return dict(precision=prep.precision, g_w=np.float32(prep.g_w), inv_lambda=prep.inv_lam,
                qw=F.pack_nibbles(qw), sw=sw, l1s=bf16_bits(prep.L1s).reshape(prep.rank, -1),
                l2=prep.L2.reshape(-1, prep.rank), bias=li.bias)


def check_weights_exact(svdq, w, exp: dict) -> None:
    """Every prepared-weight part, exported in canonical layout through the C
    ABI (svdq_export_weights), bit-exact against the oracle's preparation
    (`exp` from expected_weights)."""
    e = svdq.svdq_export_weights(w)
    assert e["g_w"] == exp["g_w"]
    assert np.array_equal(e["inv_lambda"].view(np.uint32), exp["inv_lambda"].view(np.uint32))
    assert np.array_equal(e["qw"], exp["qw"])
    sw = e["sw"] if exp["precision"] == "nvfp4" else e["sw"].view(np.uint16)
    assert np.array_equal(sw, exp["sw"])
    assert np.array_equal(e["l1s"], exp["l1s"])
    assert np.array_equal(e["l2"], exp["l2"])
    assert np.array_equal(e["bias"], exp["bias"])


def lora_scale(ol: OracleLayer, precision: str) -> np.float32:
    """The unit the kernels store lora_act in: RN32(1 / RN32(g_x g_w)) for
    NVFP4, 1 for INT4."""
    if precision != "nvfp4":
        return np.float32(1.0)
    return np.float32(1.0) / np.float32(np.float32(ol.gx) * ol.prep.g_w)


def expected_act(x: np.ndarray, prep: V.Prepared, gx) -> dict:
    """The oracle's activation codes (packed), canonical scales and
    lora_act (fp64, unscaled) for every row of x."""
    act = V.quantize_activations(x, prep, gx)
    qx = act.qx if prep.precision == "nvfp4" else F.int4_to_nibble(act.qx)
    sx = act.sx if prep.precision == "nvfp4" else act.sx.view(np.uint16)
    return dict(precision=prep.precision, qx=F.pack_nibbles(qx), sx=sx, lora_act=act.lora_act, act=act)


def e4m3_bytes(codes: np.ndarray) -> np.ndarray:
    """The E4M3 (fn) bytes of integer codes in [-8, 7], each exactly
    representable, through torch's own float8 conversion."""
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def check_act_exact(svdq, w, x: np.ndarray, ol: OracleLayer, qx, sx, la, exp: dict | None = None) -> dict:
    """Activation codes and scales of every row bit-exact against the
    oracle's quantiser (scales exported in canonical layout through the C
    ABI, svdq_export_act_scales; padded scale rows zero), and lora_act
    within the bound of the kernels' tf32 rounding."""
    M, K = x.shape
    if exp is None:
        exp = expected_act(x, ol.prep, ol.gx)
    precision = exp["precision"]
    assert np.array_equal(qx[:M * K // 2].cpu().numpy().reshape(M, K // 2), exp["qx"])
    if precision == "int4":
        # the same codes as E4M3 bytes, M rows of K, at the end of the codes buffer
        nb = svdq.svdq_act_codes_bytes(w, M)
        q8 = qx[nb - M * K:nb].cpu().numpy().reshape(M, K)
        assert np.array_equal(q8, e4m3_bytes(exp["act"].qx))
    sc = svdq.svdq_export_act_scales(w, sx, M)
    assert np.array_equal(sc if precision == "nvfp4" else sc.view(np.uint16), exp["sx"])
    mp = (M + 127) // 128 * 128
    raw = sx.cpu().numpy()
    if precision == "nvfp4":
        assert np.all(raw[tiled_scale_index(mp, K)[M:]] == 0)
    else:
        assert np.all(raw[:mp * (K // 64) * 2].view(np.float16).reshape(K // 64, mp)[:, M:] == 0)
    if la is not None:
        r = ol.prep.rank
        scale = float(lora_scale(ol, precision))
        ref = exp["lora_act"] * scale
        got = la[:M].cpu().numpy()
        mag = exp.get("lora_mag")
        if mag is None:
            mag = np.abs(x).astype(np.float64) @ np.abs(ol.prep.L1s).astype(np.float64).T
        mag = mag * scale
        assert np.all(np.abs(got[:, :r].astype(np.float64) - ref) <= 2.0 ** -11 * np.abs(ref) + 1e-5 * mag + 1e-30)
        assert np.all(got[:, r:] == 0)
    return exp


def check_y(y: np.ndarray, ref: np.ndarray, out_dtype: int, rel_f: float = 2e-3, max_abs: float = 1e-2,
            widen: float = 1.0, ref_for_scale: np.ndarray | None = None) -> None:
    """The output bar: relative Frobenius error <= rel_f; fp32 output
    (out_dtype 1): max |error| <= max_abs rms(Y*); bf16 output: per element
    |error| <= max_abs rms(Y*) + half a bf16 ulp of Y*.  `widen` scales both
    bounds (a Lipschitz activation after the layer); `ref_for_scale` is the
    pre-activation Y* whose norm and rms set them."""
    base = ref if ref_for_scale is None else ref_for_scale
    d = y.astype(np.float64) - ref
    assert np.linalg.norm(d) <= widen * rel_f * np.linalg.norm(base)
    rms = np.sqrt(np.mean(base ** 2))
    if out_dtype:
        assert np.abs(d).max() <= widen * max_abs * rms
    else:
        half_ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
        assert np.all(np.abs(d) <= widen * max_abs * rms + half_ulp)


def stack_linear_expected(args) -> dict:
    """Oracle side of one linear of the denoising stack (block `blk`, layer
    `j`), for a spawn worker: the layer inputs, the oracle's smoothing
    factor and low-rank factors (inputs of the GPU preparation too), its
    prepared weights and activation codes in canonical layout, and the fp64
    Y* of `n_rows` seeded sampled rows."""
    blk, j, n_rows, threads = args
    from threadpoolctl import threadpool_limits
    with threadpool_limits(threads):
        name = synth.STACK_LAYERS[j]
        li = synth.make_layer(name, synth.stack_seed(blk, j))
        ol = oracle_layer(li)
        ew = expected_weights(li, ol.prep)
        ea = expected_act(li.x, ol.prep, ol.gx)
        # the magnitude that bounds the lora_act rounding (see check_act_exact)
        ea["lora_mag"] = np.abs(li.x).astype(np.float64) @ np.abs(ol.prep.L1s).astype(np.float64).T
        M = li.shape.M
        rows = np.sort(np.random.default_rng(1000 + 4 * blk + j).choice(M, n_rows, replace=False))
        act = ea.pop("act")
        sub = V.ActQuant(act.qx[rows], act.sx[rows], act.lora_act[rows])
        ref = V.forward_from_codes(sub, ol.prep, ol.gx)
    ol.prep.R = None  # not needed past the preparation; keeps the transfer small
    ol.prep.qw = None
    return dict(blk=blk, j=j, name=name, x_bits=li.x_bits, w=li.w, bias_bits=li.bias_bits, bias=li.bias,
                ol=ol, exp_w=ew, exp_a=ea, rows=rows, ref=ref)
