// Warp-level walk over the split-KV partition (see common.cuh): every warp
// that needs the segment list of its engine computes it independently and
// identically, so no schedule kernel, no workspace list and no cross-warp
// hand-off is needed.
#pragma once

#include "common.cuh"

namespace mla {

struct Segment {
  int b;         // sequence
  int blk_lo;    // first logical block of the piece (within the sequence)
  int blk_hi;    // one past the last logical block
  int len;       // clamped sequence length in tokens
  int slot;      // partial slot (2p or 2p+1), or -1 when the piece is the whole sequence
  bool first_of_seq;  // this piece holds the sequence's first block
  long long pre; // concatenated index of the sequence's first block
  int nb;        // block count of the sequence
};

// Sum over b of ceil(len_b / 64); all lanes return the same value.
__device__ __forceinline__ long long warp_total_blocks(const int32_t* seq_lens, int B,
                                                       int max_blocks) {
  long long acc = 0;
  const int lane = threadIdx.x & 31;
  for (int b = lane; b < B; b += 32) {
    int L = seq_lens[b];
    L = L < 0 ? 0 : (L > max_blocks * kBlock ? max_blocks * kBlock : L);
    acc += nblocks_of(L);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

__device__ __forceinline__ int clamp_len(int L, int max_blocks) {
  return L < 0 ? 0 : (L > max_blocks * kBlock ? max_blocks * kBlock : L);
}

// Iterates the segments of engine p.  Must be driven by a whole warp (all 32
// lanes call the same methods); the returned values are warp-uniform.  With
// NBt blocks in total only min(P, NBt) engines take part.
struct SegWalker {
  const int32_t* seq_lens;
  int B, max_blocks, P, p;
  long long NBt, s, e;
  int b;            // current sequence
  long long pre;    // concatenated index of its first block
  int nb;           // its block count
  int len;
  int count;        // segments returned so far

  __device__ __noinline__ void init(const int32_t* sl, int B_, int maxb, int P_, int p_) {
    seq_lens = sl;
    B = B_;
    max_blocks = maxb;
    P = P_;
    p = p_;
    NBt = warp_total_blocks(sl, B_, maxb);
    // never more engines than blocks, so that every engine's range is
    // non-empty and the engines holding one sequence are consecutive
    if (static_cast<long long>(P) > NBt) P = static_cast<int>(NBt);
    count = 0;
    b = B;
    pre = 0;
    nb = 0;
    len = 0;
    s = e = 0;
    if (p >= P) return;
    s = range_start(p_, NBt, P);
    e = range_start(p_ + 1, NBt, P);
    if (s >= e) return;
    // find the sequence holding concatenated block s: warp scan over chunks of 32
    const int lane = threadIdx.x & 31;
    long long carry = 0;
    for (int base = 0; base < B; base += 32) {
      int bb = base + lane;
      int L = bb < B ? clamp_len(seq_lens[bb], max_blocks) : 0;
      int n = nblocks_of(L);
      long long incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        long long v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      bool hit = (n > 0) && (carry + incl > s);
      unsigned m = __ballot_sync(0xffffffffu, hit);
      if (m) {
        int src = __ffs(m) - 1;
        b = base + src;
        nb = __shfl_sync(0xffffffffu, n, src);
        len = __shfl_sync(0xffffffffu, L, src);
        pre = carry + __shfl_sync(0xffffffffu, incl, src) - nb;
        return;
      }
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }

  // Next segment; false when the engine's range is exhausted.
  __device__ __noinline__ bool next(Segment& g) {
    if (b >= B || pre >= e) return false;
    long long lo = s > pre ? s : pre;
    long long hi = e < pre + nb ? e : pre + nb;
    g.b = b;
    g.blk_lo = static_cast<int>(lo - pre);
    g.blk_hi = static_cast<int>(hi - pre);
    g.len = len;
    g.first_of_seq = (g.blk_lo == 0);
    g.pre = pre;
    g.nb = nb;
    bool whole = (g.blk_lo == 0 && g.blk_hi == nb);
    g.slot = whole ? -1 : (2 * p + (count == 0 ? 0 : 1));
    ++count;
    // advance to the next sequence with at least one block
    pre += nb;
    const int lane = threadIdx.x & 31;
    for (;;) {
      ++b;
      if (b >= B || pre >= e) break;
      int L = 0;
      if (lane == 0) L = clamp_len(seq_lens[b], max_blocks);
      L = __shfl_sync(0xffffffffu, L, 0);
      if (L > 0) {
        len = L;
        nb = nblocks_of(L);
        break;
      }
    }
    return true;
  }
};

// seq_info record of the sequence of segment g, written by the engine that
// holds the sequence's first block: (first engine, last engine, slot of the
// first engine's piece, kind).  Engines p in (first, last] hold their piece
// in slot 2p (it is their first segment).
__device__ __forceinline__ int4 seq_info_for(const Segment& g, const SegWalker& w) {
  if (g.slot < 0) return make_int4(w.p, w.p, -1, kSeqWhole);
  int p1 = engine_of(g.pre + g.nb - 1, w.NBt, w.P);
  return make_int4(w.p, p1, g.slot, kSeqCut);
}

}  // namespace mla
