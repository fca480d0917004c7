"""Unabsorbed ("naive") MLA attention in FP64 numpy.

TEST INFRASTRUCTURE ONLY.  This is the textbook form the absorbed decode must
equal exactly (up to rounding): per-head keys and values are formed from the
cached latent, RoPE is applied only to the decoupled part, and standard
softmax attention runs per head.

"Multi-Head Latent Attention: Scaling LLM Serving Throughput via Low-Rank KV
Compression" (priorstack.com), section "Empirical Gains": the content key of
head h is the up-projection of the latent, k^C_{t,h} = W^UK_h c^KV_t, the
value is v_{t,h} = W^UV_h c^KV_t, and a separate shared key k^R_t (d_h^R = 64)
carries the position; the query of head h is [q^C_h | q^R_h].  Standard
multi-head attention of each head ("Deepseek-V3 Define 1: Higher Attachment
of Head", dataforcee.us, MHA section) is softmax(q . K^T * scale) V.

RoPE ("Cords" section of the same article; "Residual & RoPE Explanation" of
"Multi-Head Latent Attention - Latent KV-Cache (DeepSeek v3)", eeumee.net):
consecutive pairs (x_{2i}, x_{2i+1}) are rotated by the angle p * theta_i at
position p, so a score depends only on the distance between query and key
positions.  Reading taken where the page is garbled: theta_i = base^(-2i/d)
with base 10000.
"""
from __future__ import annotations

import numpy as np


def rope(x: np.ndarray, pos, base: float = 10000.0) -> np.ndarray:
    """Rotate consecutive pairs of the last axis of ``x`` by pos * theta_i.
    ``pos`` broadcasts against ``x.shape[:-1]``."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    assert d % 2 == 0
    i = np.arange(d // 2, dtype=np.float64)
    theta = base ** (-2.0 * i / d)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * theta
    c, s = np.cos(ang), np.sin(ang)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = x0 * c - x1 * s
    out[..., 1::2] = x0 * s + x1 * c
    return out


def softmax_rows(s: np.ndarray) -> np.ndarray:
    """Softmax along the last axis via scipy (a library routine)."""
    from scipy.special import softmax
    return softmax(s, axis=-1)


def naive_mha(c_kv, k_r, q_nope, q_r, w_uk, w_uv, scale, q_pos=None, k_pos0=0):
    """Unabsorbed attention of one decode query against L cached tokens.

    c_kv [L,512], k_r [L,64] (before rotation), q_nope [H,128], q_r [H,64]
    (before rotation), w_uk, w_uv [H,128,512].  Keys at positions
    k_pos0..k_pos0+L-1, the query at ``q_pos`` (default the newest token).
    Returns (o [H,128] per-head attention output, scores [H,L]).
    """
    c_kv = np.asarray(c_kv, np.float64)
    k_r = np.asarray(k_r, np.float64)
    q_nope = np.asarray(q_nope, np.float64)
    q_r = np.asarray(q_r, np.float64)
    w_uk = np.asarray(w_uk, np.float64)
    w_uv = np.asarray(w_uv, np.float64)
    L = c_kv.shape[0]
    H = q_nope.shape[0]
    if q_pos is None:
        q_pos = k_pos0 + L - 1
    k_rot = rope(k_r, k_pos0 + np.arange(L))            # [L,64], shared by all heads
    q_rot = rope(q_r, np.full(H, q_pos))       # [H,64]
    o = np.empty((H, w_uv.shape[1]))
    scores = np.empty((H, L))
    for h in range(H):
        k_c = c_kv @ w_uk[h].T                 # [L,128] = W_UK[h] c_t for every t
        v = c_kv @ w_uv[h].T                   # [L,128]
        K = np.concatenate([k_c, k_rot], axis=1)        # [L,192]
        qh = np.concatenate([q_nope[h], q_rot[h]])      # [192]
        s = (K @ qh) * scale
        p = softmax_rows(s)
        o[h] = p @ v
        scores[h] = s
    return o, scores
