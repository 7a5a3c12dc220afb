"""Chained W4A4 layers: the dynamic activation tensor scale and the output
of one layer taken as the next layer's input (oracle; test infrastructure,
never called by the product path).

The pages describe the SVDQuant linear layer on its own and mention that the
original engine's architecture-specific fused kernels and modules buy more
speed than the per-module integration (mind-verse.de, "Nunchaku Lite:
Nahtlose Integration in Diffusers", the paragraph on the trade-off), and
that the remaining overhead after the 4-bit kernels is extra kernel
launches ("Eigenes Modell quantisieren" section's preceding results
paragraph).  They name no fused chain.  Readings used here:

  * Dynamic tensor scale: g_x of an NVFP4 layer is taken from the very
    activation it quantises, g_x = RN32(amax |X_hat| / 2688) (1 for a zero
    amax), X_hat = RN32(X * inv_lambda) -- the same formula as the
    calibrated scale (oracle.svdq.act_global_scale), computed per call.
  * Chained layers: the next layer's X is this layer's stored output, i.e.
    act(Y*) rounded to the output type; act is the identity or GELU in its
    tanh form (the FLUX feed-forward's activation between its up- and
    down-projection; Hendrycks and Gimpel 2016, the tanh approximation).
  * The next layer's amax is max |RN32(x * inv_lambda')| over that stored
    output: what its quantiser reads.
"""
from __future__ import annotations

import numpy as np

from . import formats as F
from . import svdq as V

GELU_K0 = np.sqrt(2.0 / np.pi)
GELU_K1 = 0.044715


def gelu_tanh(y) -> np.ndarray:
    """0.5 y (1 + tanh(sqrt(2/pi) (y + 0.044715 y^3))) in fp64."""
    y = np.asarray(y, np.float64)
    return 0.5 * y * (1.0 + np.tanh(GELU_K0 * (y + GELU_K1 * y * y * y)))


ACTIVATIONS = {"none": lambda y: np.asarray(y, np.float64), "gelu_tanh": gelu_tanh}


def round_output(y: np.ndarray, out_dtype: str) -> np.ndarray:
    """The stored layer output: bf16 (round to nearest even) or fp32."""
    if out_dtype == "bf16":
        return F.bf16_rn(np.asarray(y, np.float64)).astype(np.float32)
    return np.asarray(y, np.float64).astype(np.float32)


def act_amax(x: np.ndarray, inv_lam: np.ndarray) -> np.float32:
    """amax |X_hat| with X_hat = RN32(X * inv_lambda) (0 for an empty X)."""
    xh = V.smooth_activation(x, inv_lam)
    return np.float32(np.max(np.abs(xh))) if xh.size else np.float32(0.0)


def layer_output(x, prep: V.Prepared, activation: str = "none", g_x=None) -> np.ndarray:
    """act(Y*) in fp64 with the dynamic tensor scale when g_x is None."""
    if g_x is None and prep.precision == "nvfp4":
        g_x = V.act_global_scale(x, prep.inv_lam)
    return ACTIVATIONS[activation](V.forward(x, prep, g_x))


def chain_forward(x, prep_a: V.Prepared, prep_b: V.Prepared, activation: str = "gelu_tanh",
                  out_dtype: str = "bf16"):
    """Layer a (dynamic scale), its activation and rounded output, then
    layer b on that output with its own dynamic scale.  Returns
    (y_a stored, amax of layer b's X_hat, y_b in fp64)."""
    ya = round_output(layer_output(x, prep_a, activation), out_dtype)
    amax_b = act_amax(ya, prep_b.inv_lam)
    yb = layer_output(ya, prep_b)
    return ya, amax_b, yb
