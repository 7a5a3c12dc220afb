"""The awq_w4a16 layer: 4-bit weights, 16-bit activations (oracle; test
infrastructure: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline may import it).

Nunchaku 4-bit in Diffusers (mind-verse.de page): the second kernel family,
awq_w4a16, keeps 4-bit weights with 16-bit activations for the adaptive
normalisation and modulation projections (FLUX adanorm_single /
adanorm_zero, Qwen-Image modulation), layers that are memory-bound and
sensitive to precision; its quantization_config block ("Native
Ladefunktion") names precision int4 and group_size 64, targets such as
adaLN_modulation.1.  The page gives no formula.  Readings (listed again in
the design notes):

  * Activation-aware weight quantisation: a per-input-channel scale alpha
    (K values, from calibration; ones when none is given) moves into the
    weights, W_til = RN32(W * alpha), and out of the activations,
    X_hat = RN32(X * RN32(1 / alpha)), so that X_hat W_til^T = X W^T up to
    rounding.
  * W_til is quantised with the INT4 group-64 rule of the svdq_w4a4 INT4
    variant (oracle.quant.int4_quantize): per output row and 64-wide group
    s_h = fp16(RN32(amax / 7)), q = clamp(rint(RN32(w * RN32(1 / s_h))), -8, 7).
  * Y = X_hat (s_h q)^T + b, computed here in fp64; the activations stay in
    16 bits (no activation quantisation, no low-rank branch).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import quant as Q
from . import svdq as V


@dataclasses.dataclass
class AwqPrepared:
    q: np.ndarray        # N x K int8 in [-8, 7]
    s: np.ndarray        # N x K/64 float16
    inv_alpha: np.ndarray  # K fp32
    bias: np.ndarray     # N fp32 (bf16 values)


def prepare(w: np.ndarray, alpha: np.ndarray, bias: np.ndarray) -> AwqPrepared:
    wt = V.smooth_weight(w, alpha)
    q, s = Q.int4_quantize(wt)
    return AwqPrepared(q, s, V.inv_lambda(alpha), np.asarray(bias, np.float32))


def forward(x: np.ndarray, prep: AwqPrepared) -> np.ndarray:
    """fp64 Y* = X_hat dequant(q, s)^T + b."""
    xh = V.smooth_activation(x, prep.inv_alpha).astype(np.float64)
    return xh @ Q.int4_dequantize(prep.q, prep.s).T + prep.bias.astype(np.float64)[None, :]
