"""Seeded synthetic inputs for the absorbed MLA decode path.

This module is the one piece shared by the CUDA path and the FP64 oracle: it
only draws random numbers, rounds them to the storage types (bf16, OCP E4M3
with a per-block fp32 scale) and lays them out in the paged latent cache.  It
holds none of the method's arithmetic (no scores, no softmax, no RoPE, no
up-projection).

Shapes follow "Multi-Head Latent Attention: Scaling LLM Serving Throughput via
Low-Rank KV Compression" (priorstack.com), section "Empirical Gains": the
DeepSeek-V2 dimensions n_h = 128, d_h = 128, d_c = 512, d_h^R = 64, and one
cached row of d_c + d_h^R = 576 elements per token.

Paged layout (bf16 cache):  cache[num_blocks, 64, 576]  rows [c_kv | k_rope]
Paged layout (fp8 cache):   cache[num_blocks, 64, 512] uint8 E4M3 codes of
                            c_kv / block_scale, k_rope[num_blocks, 64, 64] bf16,
                            block_scale[num_blocks] fp32
block_table[B, max_blocks] int32: physical block of logical block j of row b,
-1 past the end.  seq_lens[B] int32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

D_C = 512          # latent width d_c
D_R = 64           # decoupled RoPE key width d_h^R
D_ROW = D_C + D_R  # one cached row
D_NOPE = 128       # per-head content query width d_h
BLOCK = 64         # tokens per cache block
FP8_MAX = 448.0    # largest finite OCP E4M3 magnitude


@dataclass
class Workload:
    name: str
    B: int
    H: int
    seq_lens: torch.Tensor            # int32 [B]
    block_table: torch.Tensor         # int32 [B, max_blocks], -1 pad
    num_blocks: int
    cache_dtype: str                  # "bf16" | "fp8"
    cache: torch.Tensor               # bf16 [NB,64,576] | uint8 [NB,64,512]
    k_rope: Optional[torch.Tensor]    # fp8 only: bf16 [NB,64,64]
    block_scale: Optional[torch.Tensor]  # fp8 only: fp32 [NB]
    q: torch.Tensor                   # bf16 [B,H,576] = [q_abs | q_rope]
    softmax_scale: float
    seed: int
    # inputs of the query absorption step (q_abs = q_nope . W_UK[h])
    q_nope: Optional[torch.Tensor] = None   # bf16 [B,H,128]
    w_uk: Optional[torch.Tensor] = None     # bf16 [H,128,512]
    # input of the output absorption step (out_h = W_UV[h] . o_latent)
    w_uv: Optional[torch.Tensor] = None     # bf16 [H,128,512]
    extras: dict = field(default_factory=dict)

    @property
    def max_blocks(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def total_tokens(self) -> int:
        return int(self.seq_lens.to(torch.int64).sum())


# The five workloads: shapes, distributions and structure as stated for the
# DeepSeek-V3 decode benchmark family.  "N(0,1)/sqrt(d)" divides by the length
# of the vector the entry belongs to (512 for c_kv / q_abs, 64 for the RoPE
# parts).
CONFIGS = {
    "tiny": dict(B=1, H=16, L=256, cache="bf16", seed=0, q_scaled=True,
                 contiguous=True),
    "v3": dict(B=64, H=128, L=4096, cache="bf16", seed=1, q_scaled=False),
    "ragged": dict(B=128, H=128, L=("uniform", 1, 8192), cache="bf16", seed=2,
                   q_scaled=False),
    "long": dict(B=4, H=128, L=131072, cache="bf16", seed=3, q_scaled=False,
                 outlier_frac=0.01, outlier_mult=8.0),
    "fp8": dict(B=64, H=128, L=16384, cache="fp8", seed=4, q_scaled=False),
}

DESCRIPTIONS = {
    "tiny": "B=1 H=16 L=256 one contiguous cache, N(0,1)/sqrt(d) inputs",
    "v3": "DeepSeek-V3 decode shape B=64 H=128 L=4096 bf16 paged cache",
    "ragged": "ragged serving batch B=128 H=128 L~U[1,8192] bf16 paged cache",
    "long": "long context B=4 H=128 L=131072 bf16 paged cache, 1% x8 outlier rows",
    "fp8": "FP8-E4M3 latent cache B=64 H=128 L=16384, per-block fp32 scale",
}


def _randn(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32) * std


def _seq_lens(spec, B: int, g: torch.Generator) -> torch.Tensor:
    if isinstance(spec, (list, tuple)) and spec and spec[0] == "uniform":
        lo, hi = int(spec[1]), int(spec[2])
        return torch.randint(lo, hi + 1, (B,), generator=g, dtype=torch.int64).to(torch.int32)
    if isinstance(spec, (list, tuple)):
        assert len(spec) == B
        return torch.tensor(list(spec), dtype=torch.int32)
    return torch.full((B,), int(spec), dtype=torch.int32)


def fp8_e4m3_encode(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 values to OCP E4M3 codes (round-to-nearest-even, saturating
    at +-448) using torch's float8_e4m3fn conversion; returns uint8 codes."""
    x = x.clamp(-FP8_MAX, FP8_MAX)
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def make(name: str, *, seed: Optional[int] = None, B: Optional[int] = None,
         H: Optional[int] = None, L=None, cache: Optional[str] = None,
         q_scaled: Optional[bool] = None, contiguous: Optional[bool] = None,
         outlier_frac: Optional[float] = None, q_std: Optional[float] = None,
         extra_blocks: int = 0, with_absorb: bool = True,
         tail_fill: Optional[float] = None, chunk_blocks: int = 2048) -> Workload:
    """Build one seeded workload.

    ``name`` picks a base config from CONFIGS; keyword overrides shrink it for
    tests.  ``q_std`` overrides the query spread (a larger value gives sharper
    softmax rows).  ``extra_blocks`` adds unused physical blocks.
    ``tail_fill`` writes that value into every cache row at or past seq_len in
    each sequence's last block (to show such rows are never read).
    """
    spec = dict(CONFIGS[name])
    if seed is not None:
        spec["seed"] = seed
    if B is not None:
        spec["B"] = B
    if H is not None:
        spec["H"] = H
    if L is not None:
        spec["L"] = L
    if cache is not None:
        spec["cache"] = cache
    if q_scaled is not None:
        spec["q_scaled"] = q_scaled
    if contiguous is not None:
        spec["contiguous"] = contiguous
    if outlier_frac is not None:
        spec["outlier_frac"] = outlier_frac

    g = torch.Generator().manual_seed(int(spec["seed"]))
    Bn, Hn = int(spec["B"]), int(spec["H"])
    seq_lens = _seq_lens(spec["L"], Bn, g)
    nblk = [(int(l) + BLOCK - 1) // BLOCK for l in seq_lens.tolist()]
    max_blocks = max(1, max(nblk) if nblk else 1)
    used = sum(nblk)
    NB = used + int(extra_blocks)
    NB = max(NB, 1)
    if spec.get("contiguous"):
        perm = torch.arange(NB, dtype=torch.int64)
    else:
        perm = torch.randperm(NB, generator=g)
    table = torch.full((Bn, max_blocks), -1, dtype=torch.int32)
    off = 0
    for b, n in enumerate(nblk):
        table[b, :n] = perm[off:off + n].to(torch.int32)
        off += n

    # queries: q_abs (d_c) and q_rope (d_r), bf16
    if q_std is not None:
        s_abs = s_rope = float(q_std)
    elif spec.get("q_scaled"):
        s_abs, s_rope = 1.0 / math.sqrt(D_C), 1.0 / math.sqrt(D_R)
    else:
        s_abs = s_rope = 1.0
    q_abs32 = _randn(g, (Bn, Hn, D_C), s_abs)
    q_rope32 = _randn(g, (Bn, Hn, D_R), s_rope)
    q = torch.cat([q_abs32, q_rope32], dim=2).to(torch.bfloat16)

    # cache, generated in chunks of physical blocks
    kind = spec["cache"]
    extras = {}
    if kind == "bf16":
        cache_t = torch.empty((NB, BLOCK, D_ROW), dtype=torch.bfloat16)
        for c0 in range(0, NB, chunk_blocks):
            c1 = min(NB, c0 + chunk_blocks)
            ck = _randn(g, (c1 - c0, BLOCK, D_C), 1.0 / math.sqrt(D_C))
            kr = _randn(g, (c1 - c0, BLOCK, D_R), 1.0 / math.sqrt(D_R))
            cache_t[c0:c1, :, :D_C] = ck.to(torch.bfloat16)
            cache_t[c0:c1, :, D_C:] = kr.to(torch.bfloat16)
        k_rope_t = None
        scale_t = None
    elif kind == "fp8":
        cache_t = torch.empty((NB, BLOCK, D_C), dtype=torch.uint8)
        k_rope_t = torch.empty((NB, BLOCK, D_R), dtype=torch.bfloat16)
        scale_t = torch.empty((NB,), dtype=torch.float32)
        for c0 in range(0, NB, chunk_blocks):
            c1 = min(NB, c0 + chunk_blocks)
            ck = _randn(g, (c1 - c0, BLOCK, D_C), 1.0 / math.sqrt(D_C))
            kr = _randn(g, (c1 - c0, BLOCK, D_R), 1.0 / math.sqrt(D_R))
            amax = ck.abs().amax(dim=(1, 2))
            sc = torch.where(amax > 0, amax / FP8_MAX, torch.ones_like(amax))
            scale_t[c0:c1] = sc
            cache_t[c0:c1] = fp8_e4m3_encode(ck / sc[:, None, None])
            k_rope_t[c0:c1] = kr.to(torch.bfloat16)
    else:
        raise ValueError(f"unknown cache kind {kind}")

    # outlier tokens: whole c_kv row times 8 (exact in bf16: a power of two)
    frac = spec.get("outlier_frac")
    if frac:
        mult = float(spec.get("outlier_mult", 8.0))
        assert kind == "bf16"
        for b in range(Bn):
            Lb = int(seq_lens[b])
            n_out = max(1, int(round(Lb * frac))) if Lb > 0 else 0
            if n_out == 0:
                continue
            toks = torch.randperm(Lb, generator=g)[:n_out]
            phys = table[b, (toks // BLOCK).long()].long()
            rows = (toks % BLOCK).long()
            cache_t[phys, rows, :D_C] = (cache_t[phys, rows, :D_C].float() * mult).to(torch.bfloat16)
        extras["outlier_mult"] = mult

    if tail_fill is not None:
        for b in range(Bn):
            Lb = int(seq_lens[b])
            if Lb % BLOCK == 0 or Lb == 0:
                continue
            blk = int(table[b, Lb // BLOCK])
            r0 = Lb % BLOCK
            if kind == "bf16":
                cache_t[blk, r0:, :] = float(tail_fill)
            else:
                cache_t[blk, r0:, :] = 0x7F  # an E4M3 NaN code
                k_rope_t[blk, r0:, :] = float(tail_fill)

    q_nope = w_uk = w_uv = None
    if with_absorb:
        # q_abs = q_nope . W_UK[h]; spreads chosen so q_abs has the same spread
        # as the directly drawn q_abs above.
        if spec.get("q_scaled"):
            qn_std, w_std = 1.0 / math.sqrt(D_NOPE), 1.0 / math.sqrt(D_C)
        else:
            qn_std, w_std = 1.0, 1.0 / math.sqrt(D_NOPE)
        q_nope = _randn(g, (Bn, Hn, D_NOPE), qn_std).to(torch.bfloat16)
        w_uk = _randn(g, (Hn, D_NOPE, D_C), w_std).to(torch.bfloat16)
        # drawn last, so every earlier draw is unchanged by its presence
        w_uv = _randn(g, (Hn, D_NOPE, D_C), 1.0 / math.sqrt(D_C)).to(torch.bfloat16)

    return Workload(name=name, B=Bn, H=Hn, seq_lens=seq_lens, block_table=table,
                    num_blocks=NB, cache_dtype=kind, cache=cache_t, k_rope=k_rope_t,
                    block_scale=scale_t, q=q, softmax_scale=1.0 / math.sqrt(D_NOPE + D_R),
                    seed=int(spec["seed"]), q_nope=q_nope, w_uk=w_uk, w_uv=w_uv, extras=extras)


def relocate(w: Workload, seed: int) -> Workload:
    """Same logical cache, different physical placement: a new random block
    permutation (block_table and cache rows move together)."""
    g = torch.Generator().manual_seed(int(seed))
    NB = w.num_blocks
    new_of_old = torch.randperm(NB, generator=g)
    old_of_new = torch.empty_like(new_of_old)
    old_of_new[new_of_old] = torch.arange(NB)
    table = w.block_table.clone()
    m = table >= 0
    table[m] = new_of_old[table[m].long()].to(torch.int32)
    cache = w.cache[old_of_new]
    k_rope = w.k_rope[old_of_new] if w.k_rope is not None else None
    scale = w.block_scale[old_of_new] if w.block_scale is not None else None
    return Workload(name=w.name + "+reloc", B=w.B, H=w.H, seq_lens=w.seq_lens.clone(),
                    block_table=table, num_blocks=NB, cache_dtype=w.cache_dtype,
                    cache=cache, k_rope=k_rope, block_scale=scale, q=w.q.clone(),
                    softmax_scale=w.softmax_scale, seed=w.seed, q_nope=w.q_nope,
                    w_uk=w.w_uk, extras=dict(w.extras))


def raw_tiny_fp32(seed: int = 0, H: int = 16, L: int = 256):
    """Pre-rounding fp32 draws for the small naive-vs-absorbed check:
    c_kv [L,512], pre-rotation k_r [L,64], q_nope [H,128], pre-rotation q_r
    [H,64], W_UK and W_UV [H,128,512]."""
    g = torch.Generator().manual_seed(int(seed) + 1000)
    return dict(
        c_kv=_randn(g, (L, D_C), 1.0 / math.sqrt(D_C)),
        k_r=_randn(g, (L, D_R), 1.0 / math.sqrt(D_R)),
        q_nope=_randn(g, (H, D_NOPE), 1.0 / math.sqrt(D_NOPE)),
        q_r=_randn(g, (H, D_R), 1.0 / math.sqrt(D_R)),
        w_uk=_randn(g, (H, D_NOPE, D_C), 1.0 / math.sqrt(D_C)),
        w_uv=_randn(g, (H, D_NOPE, D_C), 1.0 / math.sqrt(D_C)),
    )
