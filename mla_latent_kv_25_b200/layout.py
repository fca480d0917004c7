"""Host-side sizes of the paged latent cache and of one decode step.

Per-token cache sizes follow "Multi-Head Latent Attention: Scaling LLM
Serving Throughput via Low-Rank KV Compression" (priorstack.com), section
"Empirical Gains": MHA keeps 2*n_h*d_h elements per token per layer, GQA
2*n_g*d_h, MQA 2*d_h, and MLA only the latent plus the decoupled RoPE key,
d_c + d_h^R.
"""
from __future__ import annotations

D_C = 512
D_R = 64
D_ROW = D_C + D_R
BLOCK = 64


def cache_elements_per_token(kind: str, *, n_h: int = 128, d_h: int = 128, d_c: int = D_C,
                             d_h_r: int = D_R, n_g: int = 1, layers: int = 1) -> int:
    """Cached elements per token (times ``layers``) for one attention kind."""
    if kind == "mha":
        return 2 * n_h * d_h * layers
    if kind == "gqa":
        return 2 * n_g * d_h * layers
    if kind == "mqa":
        return 2 * d_h * layers
    if kind == "mla":
        return (d_c + d_h_r) * layers
    raise ValueError(kind)


def equivalent_gqa_groups(*, d_h: int = 128, d_c: int = D_C, d_h_r: int = D_R) -> float:
    """The GQA group count whose cache per token equals MLA's."""
    return (d_c + d_h_r) / (2.0 * d_h)


def bytes_per_token(cache_dtype: str) -> int:
    """HBM bytes of one cached row: bf16 [c_kv | k_rope] = 1152 B; fp8 cache:
    512 one-byte E4M3 codes plus the 64 bf16 RoPE values = 640 B."""
    if cache_dtype == "bf16":
        return D_ROW * 2
    if cache_dtype == "fp8":
        return D_C + D_R * 2
    raise ValueError(cache_dtype)


def decode_algorithmic_bytes(total_tokens: int, B: int, H: int, cache_dtype: str,
                             num_blocks_read: int = 0) -> int:
    """Bytes a decode call must move at minimum: every cached row of every
    actual token once, the packed query [B,H,576] bf16, the output
    [B,H,512] bf16 and lse [B,H] fp32 (plus one fp32 scale per block read
    for the fp8 cache).  Split-KV workspace traffic is not counted."""
    b = total_tokens * bytes_per_token(cache_dtype)
    b += B * H * D_ROW * 2
    b += B * H * (D_C * 2 + 4)
    if cache_dtype == "fp8":
        b += num_blocks_read * 4
    return b


def decode_flops(total_tokens: int, H: int) -> int:
    """2*H*sum(L)*(576 + 512): the QK^T contraction over the whole row and the
    PV contraction over the latent."""
    return 2 * H * total_tokens * (D_ROW + D_C)


def absorb_algorithmic_bytes(B: int, H: int) -> int:
    """q_nope [B,H,128] + W_UK [H,128,512] + q_rope [B,H,64] read, packed
    q [B,H,576] written; all bf16."""
    return 2 * (B * H * 128 + H * 128 * D_C + B * H * D_R + B * H * D_ROW)


def absorb_flops(B: int, H: int) -> int:
    return 2 * B * H * 128 * D_C
