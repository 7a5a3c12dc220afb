"""Helpers shared by the GPU parity tests: uploading the seeded inputs,
running the CUDA path through the C ABI, running the oracle on the same
inputs, and the scale-layout index map documented in include/svdq.h."""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import synth
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
    qx = aligned_empty(M * K // 2)
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
