"""The attention prologue of the fused QKV projection (oracle; test
infrastructure: only tests/, __graft_entry__.smoke() and bench.py's CPU
baseline may import it).

Nunchaku 4-bit in Diffusers, section "Quantisierung von Modellen mit
strukturellen Umschreibungen": the FLUX to_q / to_k / to_v projections are
merged into one quantised to_qkv module because the fused operator handles
the QKV projection, the Q/K normalisation and the rotary embeddings
together.  The page names the three steps and nothing more.  Readings
(listed again in the design notes), following the FLUX attention block the
page refers to:

  * Y = [Q | K | V] along the output features, each `heads * head_dim`
    wide; head h of Q is columns h*head_dim .. +head_dim-1 of Q.
  * Q/K normalisation is RMS normalisation over each head's head_dim
    values with a learned per-dimension weight, one for Q and one for K:
        q_n[d] = q[d] / sqrt(mean_d(q^2) + eps) * w_q[d].
  * The rotary embedding comes after the normalisation and acts on the
    adjacent pairs (2i, 2i+1) of every head of Q and of K, with per-token
    tables cos[m, i], sin[m, i] (i < head_dim/2) given as inputs (the
    positional frequencies are computed outside the layer):
        (a, b) -> (a cos - b sin, a sin + b cos).
  * V passes unchanged.

Everything here is fp64.
"""
from __future__ import annotations

import numpy as np


def rms_norm_heads(y: np.ndarray, weight: np.ndarray, head_dim: int, eps: float) -> np.ndarray:
    """RMS normalisation of every head_dim-wide slice of every row of y
    (M x heads*head_dim), scaled by weight[d] (head_dim values)."""
    y = np.asarray(y, np.float64)
    m, n = y.shape
    assert n % head_dim == 0
    h = y.reshape(m, n // head_dim, head_dim)
    ms = np.mean(h * h, axis=2, keepdims=True)
    out = h / np.sqrt(ms + float(eps)) * np.asarray(weight, np.float64)[None, None, :]
    return out.reshape(m, n)


def rotary_pairs(y: np.ndarray, cos: np.ndarray, sin: np.ndarray, head_dim: int) -> np.ndarray:
    """Rotates the pairs (2i, 2i+1) of every head of every row m by the
    angle whose cosine and sine are cos[m, i], sin[m, i]."""
    y = np.asarray(y, np.float64)
    m, n = y.shape
    assert n % head_dim == 0 and head_dim % 2 == 0
    c = np.asarray(cos, np.float64).reshape(m, 1, head_dim // 2)
    s = np.asarray(sin, np.float64).reshape(m, 1, head_dim // 2)
    h = y.reshape(m, n // head_dim, head_dim // 2, 2)
    a, b = h[..., 0], h[..., 1]
    out = np.empty_like(h)
    out[..., 0] = a * c - b * s
    out[..., 1] = a * s + b * c
    return out.reshape(m, n)


def qkv_prologue(y: np.ndarray, heads: int, head_dim: int, norm_q: np.ndarray, norm_k: np.ndarray,
                 cos: np.ndarray, sin: np.ndarray, eps: float) -> np.ndarray:
    """[Q | K | V] -> [rope(norm_q(Q)) | rope(norm_k(K)) | V]."""
    y = np.asarray(y, np.float64)
    w = heads * head_dim
    assert y.shape[1] == 3 * w
    out = y.copy()
    out[:, :w] = rotary_pairs(rms_norm_heads(y[:, :w], norm_q, head_dim, eps), cos, sin, head_dim)
    out[:, w:2 * w] = rotary_pairs(rms_norm_heads(y[:, w:2 * w], norm_k, head_dim, eps), cos, sin, head_dim)
    return out


def rope_tables(positions: np.ndarray, head_dim: int, theta: float = 10000.0):
    """fp32 cos/sin tables for integer token positions (M values): angle
    positions[m] * theta^(-2i/head_dim) for pair i.  A convenience for
    building test inputs; the layer itself takes the tables as given."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    ang = np.asarray(positions, np.float64)[:, None] * theta ** (-2.0 * i / head_dim)[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
