"""Writers of the paged latent cache, in plain numpy (FP64 where arithmetic).

TEST INFRASTRUCTURE ONLY: the tests are the only callers; nothing here is
shared with, or called by, the CUDA path.

* ``append``: the row a new token adds to the cache ("Multi-Head Latent
  Attention: Scaling LLM Serving Throughput via Low-Rank KV Compression",
  priorstack.com, "Empirical Gains": MLA caches only the compressed latent
  c^KV next to the decoupled key k^R; the RoPE rotation is applied to k^R
  before caching — "Multi-Head Latent Attention - Latent KV-Cache (DeepSeek
  v3)", eeumee.net, RoPE applied in FP32).  Row = [c_kv | RoPE(k_r, pos)],
  placed at physical block block_table[b, pos // 64], row pos % 64.
* ``quantize_e4m3_blocks``: the FP8 cache of "FP8/FP32 Mixed Precision"
  (eeumee.net): per 64-token block, scale = amax / 448 (1 when the block is
  all zeros), codes = c_kv / scale rounded to the nearest OCP E4M3 value
  (ties to the even code, saturating at +-448).  The divisions are taken in
  fp32, the precision the GPU takes them in, because they decide the codes.
"""
from __future__ import annotations

import numpy as np

from . import naive

BLOCK, D_C, D_R = 64, 512, 64
E4M3_MAX = 448.0


def _bf16_to_f64(u16: np.ndarray) -> np.ndarray:
    return (np.asarray(u16, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def append(c_kv, k_r, seq_idx, pos, block_table):
    """Rows a batch of new tokens writes: returns (block ids, row ids, rows)
    with rows [T, 576] float64 = [c_kv | RoPE(k_r, pos)].  Inputs bf16 bit
    patterns (uint16): c_kv [T,512], k_r [T,64]; int seq_idx [T], pos [T];
    block_table [B, max_blocks]."""
    ck = _bf16_to_f64(c_kv)
    kr = _bf16_to_f64(k_r)
    pos = np.asarray(pos, np.int64)
    seq_idx = np.asarray(seq_idx, np.int64)
    table = np.asarray(block_table)
    blocks = table[seq_idx, pos // BLOCK].astype(np.int64)
    rows = np.concatenate([ck, naive.rope(kr, pos)], axis=1)
    return blocks, (pos % BLOCK).astype(np.int64), rows


def _e4m3_values() -> tuple[np.ndarray, np.ndarray]:
    """Every finite OCP E4M3 code (NaN codes 0x7F and 0xFF excluded) with its
    value, decoded from the format's definition: 1 sign, 4 exponent bits
    (bias 7), 3 mantissa bits; exponent 0 is subnormal (m/8 * 2^-6)."""
    codes, vals = [], []
    for c in range(256):
        e, m, s = (c >> 3) & 15, c & 7, -1.0 if c & 128 else 1.0
        if e == 15 and m == 7:
            continue
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        codes.append(c)
        vals.append(s * v)
    return np.array(codes, np.uint8), np.array(vals, np.float64)


_CODES, _VALS = _e4m3_values()


def e4m3_round(y: np.ndarray) -> np.ndarray:
    """Nearest E4M3 code of each value (saturating at +-448).  Ties between
    two codes go to the even mantissa; zero keeps the sign of the input.
    Brute force over the 254 finite codes."""
    y = np.clip(np.asarray(y, np.float64), -E4M3_MAX, E4M3_MAX)
    flat = y.reshape(-1)
    out = np.empty(flat.shape, np.uint8)
    even = ((_CODES & 1) == 0).astype(np.int64)
    neg_code = ((_CODES & 128) != 0)
    for a in range(0, flat.size, 4096):
        v = flat[a:a + 4096]
        d = np.abs(_VALS[None, :] - v[:, None])
        cand = d == d.min(axis=1, keepdims=True)
        same_sign = (neg_code[None, :] == np.signbit(v)[:, None]).astype(np.int64)
        score = np.where(cand, 1 + 2 * even[None, :] + same_sign, 0)
        out[a:a + 4096] = _CODES[np.argmax(score, axis=1)]
    return out.reshape(y.shape)


def quantize_e4m3_blocks(c_kv_blocks):
    """c_kv_blocks: bf16 bit patterns [n, 64, 512].  Returns (codes uint8
    [n,64,512], scale float32 [n])."""
    x = _bf16_to_f64(c_kv_blocks).astype(np.float32)
    n = x.shape[0]
    codes = np.empty(x.shape, np.uint8)
    scale = np.empty(n, np.float32)
    for i in range(n):
        amax = np.float32(np.max(np.abs(x[i])))
        sc = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
        scale[i] = sc
        codes[i] = e4m3_round((x[i] / sc).astype(np.float32))
    return codes, scale
