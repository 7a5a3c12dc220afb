"""Thin Python binding of libsvdq (include/svdq.h).

Argument marshalling only: tensors are passed as device pointers, streams as
cudaStream_t handles; every step of the layer runs in the library's CUDA
kernels.  The functions keep the C names.  A missing library is an error
(there is no fallback path).
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsvdq.so")

SVDQ_NVFP4 = 0
SVDQ_INT4 = 1
SVDQ_AWQ_W4A16 = 2
SVDQ_OUT_BF16 = 0
SVDQ_OUT_F32 = 1
SVDQ_ACT_NONE = 0
SVDQ_ACT_GELU_TANH = 1

STATUS_NAMES = {
    0: "SVDQ_OK",
    1: "SVDQ_ERR_INVALID_ARG",
    2: "SVDQ_ERR_SHAPE",
    3: "SVDQ_ERR_ALIGNMENT",
    4: "SVDQ_ERR_UNSUPPORTED_DEVICE",
    5: "SVDQ_ERR_CUDA",
    6: "SVDQ_ERR_TIMEOUT",
    7: "SVDQ_ERR_WORKSPACE",
}


class SVDQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)} ({svdq_status_string(self.status)})")


class LayerDesc(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("rank", ctypes.c_int32),
                ("precision", ctypes.c_int32), ("group_size", ctypes.c_int32)]


class WeightsView(ctypes.Structure):
    _fields_ = [("K", ctypes.c_int32), ("N", ctypes.c_int32), ("rank", ctypes.c_int32), ("rank_pad", ctypes.c_int32),
                ("precision", ctypes.c_int32), ("group_size", ctypes.c_int32), ("n_pad", ctypes.c_int32),
                ("g_w", ctypes.c_float), ("qw", ctypes.c_void_p), ("sw", ctypes.c_void_p),
                ("sw_bytes", ctypes.c_size_t), ("l1s", ctypes.c_void_p), ("l2", ctypes.c_void_p),
                ("inv_lambda", ctypes.c_void_p), ("bias", ctypes.c_void_p)]


class WeightsExport(ctypes.Structure):
    _fields_ = [("qw", ctypes.c_void_p), ("sw", ctypes.c_void_p), ("l1s", ctypes.c_void_p), ("l2", ctypes.c_void_p),
                ("inv_lambda", ctypes.c_void_p), ("bias", ctypes.c_void_p), ("g_w", ctypes.c_void_p)]


class QkvPrologue(ctypes.Structure):
    """svdq_qkv_prologue: the attention prologue of a fused QKV projection
    (per-head RMS normalisation of Q and K with weights norm_q / norm_k,
    rotary embedding with cos / sin tables stored frequency-major,
    head_dim/2 x M: entry (i, m) for pair i of token m)."""
    _fields_ = [("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("eps", ctypes.c_float),
                ("norm_q", ctypes.c_void_p), ("norm_k", ctypes.c_void_p), ("rope_cos", ctypes.c_void_p),
                ("rope_sin", ctypes.c_void_p)]


def make_qkv_prologue(heads: int, norm_q, norm_k, rope_cos, rope_sin, eps: float = 1e-6,
                      head_dim: int = 128) -> QkvPrologue:
    """The caller keeps the four device tensors alive while the struct is used."""
    return QkvPrologue(heads, head_dim, float(eps), _ptr(norm_q), _ptr(norm_k), _ptr(rope_cos), _ptr(rope_sin))


class EpilogueNext(ctypes.Structure):
    _fields_ = [("activation", ctypes.c_int32), ("next_inv_lambda", ctypes.c_void_p), ("next_amax", ctypes.c_void_p)]


def make_epilogue_next(activation: int = SVDQ_ACT_NONE, next_inv_lambda=None, next_amax=None) -> EpilogueNext:
    """The caller keeps the device tensors alive while the struct is used."""
    return EpilogueNext(int(activation), _ptr(next_inv_lambda), _ptr(next_amax))


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int32
_F = ctypes.c_float
_Z = ctypes.c_size_t
_SIGS = {
    "svdq_status_string": (ctypes.c_char_p, [_I]),
    "svdq_check_device": (_I, [ctypes.c_int]),
    "svdq_smoothing_lambda": (_I, [_P, _I, _P, _I, _I, _P, _P, _P]),
    "svdq_weights_bytes": (_Z, [ctypes.POINTER(LayerDesc)]),
    "svdq_prepare_weights": (_I, [ctypes.POINTER(LayerDesc), _P, _P, _P, _P, _P, _P, _Z, ctypes.POINTER(_P), _P]),
    "svdq_weights_destroy": (None, [_P]),
    "svdq_weights_get_view": (_I, [_P, ctypes.POINTER(WeightsView)]),
    "svdq_export_weights": (_I, [_P, ctypes.POINTER(WeightsExport), _P]),
    "svdq_export_act_scales": (_I, [_P, _P, _I, _P, _P]),
    "svdq_act_global_scale": (_I, [_P, _P, _I, _P, _P]),
    "svdq_act_amax": (_I, [_P, _P, _I, _P, _P]),
    "svdq_act_scale_bytes": (_Z, [_P, _I]),
    "svdq_act_codes_bytes": (_Z, [_P, _I]),
    "svdq_quantize_act_lora_down": (_I, [_P, _P, _I, _F, _P, _P, _P, _P]),
    "svdq_quantize_act_lora_down_dyn": (_I, [_P, _P, _I, _P, _P, _P, _P, _P]),
    "svdq_w4a4_gemm_lora_up": (_I, [_P, _P, _P, _F, _P, _I, _P, _I, _P]),
    "svdq_w4a4_gemm_lora_up_dyn": (_I, [_P, _P, _P, _P, _P, _I, ctypes.POINTER(QkvPrologue),
                                        ctypes.POINTER(EpilogueNext), _P, _I, _P]),
    "svdq_linear_forward_dyn": (_I, [_P, _P, _I, _P, ctypes.POINTER(QkvPrologue), ctypes.POINTER(EpilogueNext), _P,
                                     _I, _P, _Z, _P]),
    "svdq_w4a4_gemm_lora_up_qkv": (_I, [_P, _P, _P, _F, _P, _I, ctypes.POINTER(QkvPrologue), _P, _I, _P]),
    "svdq_workspace_bytes": (_Z, [_P, _I]),
    "svdq_linear_forward": (_I, [_P, _P, _I, _F, _P, _I, _P, _Z, _P]),
    "svdq_linear_forward_qkv": (_I, [_P, _P, _I, _F, ctypes.POINTER(QkvPrologue), _P, _I, _P, _Z, _P]),
    "svdq_linear_forward_noalloc": (_I, [_P, _P, _I, _F, _P, _I, _P]),
    "svdq_awq_w4a16_forward": (_I, [_P, _P, _I, _P, _I, _P]),
    "svdq_lowrank_workspace_bytes": (_Z, [_I, _I]),
    "svdq_lowrank_factors": (_I, [_P, _I, _I, _P, _I, _I, _I, _P, _P, _P, _P, _Z, _P]),
    "svdq_device_status": (_I, [_P, _P]),
    "svdq_selftest_bounded_wait": (_I, [_P]),
}


def load_library() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libsvdq.so is not built ({LIB_PATH}); run `python -m bit_diffusion_transformer_svdq_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _ptr(t) -> int | None:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != 0:
        raise SVDQError(status, where)


def svdq_status_string(status: int) -> str:
    return load_library().svdq_status_string(int(status)).decode()


def svdq_check_device(device: int = 0) -> int:
    return load_library().svdq_check_device(int(device))


def make_desc(K: int, N: int, rank: int, precision: int = SVDQ_NVFP4) -> LayerDesc:
    return LayerDesc(K, N, rank, precision, 16 if precision == SVDQ_NVFP4 else 64)


def svdq_weights_bytes(desc: LayerDesc) -> int:
    return load_library().svdq_weights_bytes(ctypes.byref(desc))


def svdq_smoothing_lambda(X: torch.Tensor, W: torch.Tensor, lam: torch.Tensor, scratch: torch.Tensor, stream=None):
    M, K = X.shape
    N = W.shape[0]
    _check(load_library().svdq_smoothing_lambda(_ptr(X), M, _ptr(W), N, K, _ptr(lam), _ptr(scratch), _stream(stream)),
           "svdq_smoothing_lambda")


class Weights:
    """Owns the host handle of prepared weights and keeps the caller's
    device storage tensor alive alongside it."""

    def __init__(self, handle: int, storage: torch.Tensor, desc: LayerDesc):
        self.handle = handle
        self.storage = storage
        self.desc = desc

    @property
    def _as_parameter_(self):
        return self.handle

    def view(self) -> WeightsView:
        v = WeightsView()
        _check(load_library().svdq_weights_get_view(self.handle, ctypes.byref(v)), "svdq_weights_get_view")
        return v

    def close(self) -> None:
        if self.handle:
            load_library().svdq_weights_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def svdq_prepare_weights(desc: LayerDesc, W, lam, L1, L2, bias, storage: torch.Tensor, stream=None) -> Weights:
    out = ctypes.c_void_p()
    _check(load_library().svdq_prepare_weights(ctypes.byref(desc), _ptr(W), _ptr(lam), _ptr(L1), _ptr(L2), _ptr(bias),
                                               _ptr(storage), storage.numel() * storage.element_size(),
                                               ctypes.byref(out), _stream(stream)), "svdq_prepare_weights")
    return Weights(out.value, storage, desc)


def svdq_export_weights(w: Weights, stream=None) -> dict:
    """Canonical host copies of prepared weights (numpy arrays): qw (N x K/2
    packed codes), sw (N x K/16 E4M3 bytes, or N x K/64 float16), l1s
    (rank x K bf16 bits), l2 (N x rank fp32), inv_lambda (K), bias (N), g_w."""
    import numpy as np
    v = w.view()
    K, N, r = v.K, v.N, v.rank
    out = dict(qw=np.empty((N, K // 2), np.uint8),
               sw=np.empty((N, K // 16), np.uint8) if v.precision == SVDQ_NVFP4 else np.empty((N, K // 64), np.float16),
               l1s=np.empty((r, K), np.uint16), l2=np.empty((N, r), np.float32),
               inv_lambda=np.empty(K, np.float32), bias=np.empty(N, np.float32), g_w=np.empty(1, np.float32))
    ex = WeightsExport(*(out[k].ctypes.data if out[k].size else None
                         for k in ("qw", "sw", "l1s", "l2", "inv_lambda", "bias", "g_w")))
    _check(load_library().svdq_export_weights(w.handle, ctypes.byref(ex), _stream(stream)), "svdq_export_weights")
    out["g_w"] = np.float32(out["g_w"][0])
    return out


def svdq_export_act_scales(w: Weights, sx, M: int, stream=None):
    """Canonical host copy of activation scales: M x K/16 E4M3 bytes (NVFP4)
    or M x K/64 float16 (INT4)."""
    import numpy as np
    v = w.view()
    out = np.empty((M, v.K // 16), np.uint8) if v.precision == SVDQ_NVFP4 else np.empty((M, v.K // 64), np.float16)
    _check(load_library().svdq_export_act_scales(w.handle, _ptr(sx), M, out.ctypes.data if out.size else None,
                                                 _stream(stream)), "svdq_export_act_scales")
    return out


def svdq_act_global_scale(w: Weights, X: torch.Tensor, g_x: torch.Tensor, stream=None) -> None:
    _check(load_library().svdq_act_global_scale(w.handle, _ptr(X), X.shape[0], _ptr(g_x), _stream(stream)),
           "svdq_act_global_scale")


def svdq_act_amax(w: Weights, X: torch.Tensor, amax: torch.Tensor, stream=None) -> None:
    _check(load_library().svdq_act_amax(w.handle, _ptr(X), X.shape[0], _ptr(amax), _stream(stream)), "svdq_act_amax")


def svdq_act_scale_bytes(w: Weights, M: int) -> int:
    return load_library().svdq_act_scale_bytes(w.handle, M)


def svdq_act_codes_bytes(w: Weights, M: int) -> int:
    return load_library().svdq_act_codes_bytes(w.handle, M)


def svdq_workspace_bytes(w: Weights, M: int) -> int:
    return load_library().svdq_workspace_bytes(w.handle, M)


def svdq_quantize_act_lora_down(w: Weights, X, M: int, g_x: float, qx, sx, lora_act, stream=None) -> None:
    _check(load_library().svdq_quantize_act_lora_down(w.handle, _ptr(X), M, float(g_x), _ptr(qx), _ptr(sx),
                                                      _ptr(lora_act), _stream(stream)), "svdq_quantize_act_lora_down")


def svdq_quantize_act_lora_down_dyn(w: Weights, X, M: int, x_amax, qx, sx, lora_act, stream=None) -> None:
    _check(load_library().svdq_quantize_act_lora_down_dyn(w.handle, _ptr(X), M, _ptr(x_amax), _ptr(qx), _ptr(sx),
                                                          _ptr(lora_act), _stream(stream)),
           "svdq_quantize_act_lora_down_dyn")


def _byref(s):
    return None if s is None else ctypes.byref(s)


def svdq_w4a4_gemm_lora_up_dyn(w: Weights, qx, sx, x_amax, lora_act, M: int, Y, pro: QkvPrologue | None = None,
                               epi: EpilogueNext | None = None, out_dtype: int = SVDQ_OUT_BF16, stream=None) -> None:
    _check(load_library().svdq_w4a4_gemm_lora_up_dyn(w.handle, _ptr(qx), _ptr(sx), _ptr(x_amax), _ptr(lora_act), M,
                                                     _byref(pro), _byref(epi), _ptr(Y), out_dtype, _stream(stream)),
           "svdq_w4a4_gemm_lora_up_dyn")


def svdq_linear_forward_dyn(w: Weights, X, M: int, x_amax, Y, workspace, ws_bytes: int,
                            pro: QkvPrologue | None = None, epi: EpilogueNext | None = None,
                            out_dtype: int = SVDQ_OUT_BF16, stream=None) -> None:
    """The layer with the dynamic tensor scale; x_amax None computes it
    from X inside the call (an amax pass into the workspace)."""
    _check(load_library().svdq_linear_forward_dyn(w.handle, _ptr(X), M, _ptr(x_amax), _byref(pro), _byref(epi),
                                                  _ptr(Y), out_dtype, _ptr(workspace), ws_bytes, _stream(stream)),
           "svdq_linear_forward_dyn")


def svdq_w4a4_gemm_lora_up(w: Weights, qx, sx, g_x: float, lora_act, M: int, Y, out_dtype: int = SVDQ_OUT_BF16,
                           stream=None) -> None:
    _check(load_library().svdq_w4a4_gemm_lora_up(w.handle, _ptr(qx), _ptr(sx), float(g_x), _ptr(lora_act), M, _ptr(Y),
                                                 out_dtype, _stream(stream)), "svdq_w4a4_gemm_lora_up")


def svdq_w4a4_gemm_lora_up_qkv(w: Weights, qx, sx, g_x: float, lora_act, M: int, pro: QkvPrologue, Y,
                               out_dtype: int = SVDQ_OUT_BF16, stream=None) -> None:
    _check(load_library().svdq_w4a4_gemm_lora_up_qkv(w.handle, _ptr(qx), _ptr(sx), float(g_x), _ptr(lora_act), M,
                                                     ctypes.byref(pro), _ptr(Y), out_dtype, _stream(stream)),
           "svdq_w4a4_gemm_lora_up_qkv")


def svdq_linear_forward_qkv(w: Weights, X, M: int, g_x: float, pro: QkvPrologue, Y, workspace, ws_bytes: int,
                            out_dtype: int = SVDQ_OUT_BF16, stream=None) -> None:
    _check(load_library().svdq_linear_forward_qkv(w.handle, _ptr(X), M, float(g_x), ctypes.byref(pro), _ptr(Y),
                                                  out_dtype, _ptr(workspace), ws_bytes, _stream(stream)),
           "svdq_linear_forward_qkv")


def svdq_linear_forward(w: Weights, X, M: int, g_x: float, Y, workspace, ws_bytes: int,
                        out_dtype: int = SVDQ_OUT_BF16, stream=None) -> None:
    _check(load_library().svdq_linear_forward(w.handle, _ptr(X), M, float(g_x), _ptr(Y), out_dtype, _ptr(workspace),
                                              ws_bytes, _stream(stream)), "svdq_linear_forward")


def svdq_linear_forward_noalloc(w: Weights, X, M: int, g_x: float, Y, out_dtype: int = SVDQ_OUT_BF16,
                                stream=None) -> None:
    """The forward for callers that cannot allocate device memory: the
    intermediates live in the library's own static device scratch (16 MiB;
    larger M raises SVDQ_ERR_WORKSPACE).  Calls that overlap on the GPU race
    on that scratch."""
    _check(load_library().svdq_linear_forward_noalloc(w.handle, _ptr(X), M, float(g_x), _ptr(Y), out_dtype,
                                                      _stream(stream)), "svdq_linear_forward_noalloc")


def svdq_awq_w4a16_forward(w: Weights, X, M: int, Y, out_dtype: int = SVDQ_OUT_BF16, stream=None) -> None:
    """The awq_w4a16 layer: Y = X_hat dequant(q, s)^T + b for weights
    prepared with precision SVDQ_AWQ_W4A16 (lambda = the AWQ channel scale)."""
    _check(load_library().svdq_awq_w4a16_forward(w.handle, _ptr(X), M, _ptr(Y), out_dtype, _stream(stream)),
           "svdq_awq_w4a16_forward")


def svdq_lowrank_workspace_bytes(N: int, K: int) -> int:
    return load_library().svdq_lowrank_workspace_bytes(N, K)


def svdq_lowrank_factors(W, lam, rank: int, omega, L1, L2, workspace, oversample: int = 16, power_steps: int = 4,
                         stream=None) -> None:
    """Rank-`rank` factors of the smoothed weight (W: N x K fp32, lam: K,
    omega: N x (rank + oversample) fp32 start block) into L1 (rank x K bf16
    bits) and L2 (N x rank bf16 bits)."""
    N, K = W.shape
    _check(load_library().svdq_lowrank_factors(_ptr(W), N, K, _ptr(lam), rank, oversample, power_steps, _ptr(omega),
                                               _ptr(L1), _ptr(L2), _ptr(workspace),
                                               workspace.numel() * workspace.element_size(), _stream(stream)),
           "svdq_lowrank_factors")


def svdq_device_status(w: Weights, stream=None) -> int:
    return load_library().svdq_device_status(w.handle, _stream(stream))


def svdq_selftest_bounded_wait(stream=None) -> int:
    """Runs the bounded-wait self-test kernel; a healthy library returns
    SVDQ_ERR_TIMEOUT (6) after about two seconds."""
    return load_library().svdq_selftest_bounded_wait(_stream(stream))


# ----------------------------------------------------------------- helpers
# Allocation-only conveniences (torch owns the device memory).

def prepare_layer(W: torch.Tensor, lam: torch.Tensor, L1: torch.Tensor | None, L2: torch.Tensor | None,
                  bias: torch.Tensor | None, rank: int, precision: int = SVDQ_NVFP4, stream=None) -> Weights:
    """W (N x K fp32), lam (K fp32), L1 (rank x K bf16), L2 (N x rank bf16),
    bias (N bf16), all on the current CUDA device."""
    N, K = W.shape
    desc = make_desc(K, N, rank, precision)
    nbytes = svdq_weights_bytes(desc)
    if nbytes == 0:
        raise SVDQError(2, "svdq_weights_bytes")
    storage = torch.empty(nbytes + 1024, dtype=torch.uint8, device=W.device)
    off = (-storage.data_ptr()) % 1024
    storage = storage[off:off + nbytes]
    return svdq_prepare_weights(desc, W, lam, L1, L2, bias, storage, stream)


def alloc_workspace(w: Weights | None, M: int, device, nbytes: int | None = None) -> torch.Tensor:
    """A 1024-aligned device workspace of svdq_workspace_bytes(w, M) bytes
    (or `nbytes`, e.g. the largest over several layers sharing it, or the
    factoriser's svdq_lowrank_workspace_bytes)."""
    n = svdq_workspace_bytes(w, M) if nbytes is None else nbytes
    buf = torch.empty(n + 1024, dtype=torch.uint8, device=device)
    off = (-buf.data_ptr()) % 1024
    return buf[off:off + n]
