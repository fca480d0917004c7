// Host-side planning of an fp8-cache decode: the widened bf16 copy's place in
// the workspace and the groups of sequences a call runs in.  Shared by api.cu
// and the host checker in tests/partition_check.cu.
#pragma once

#include <stddef.h>

#include "common.cuh"

namespace mla {

// The fp8 cache's widened bf16 copy, placed after the split-KV workspace:
// a scratch block table int32 [B * max_blocks] and a dense bf16 cache
// [B * max_blocks, 64, 576] (block b * max_blocks + j holds logical block j
// of sequence b).  Its block ids and TMA row coordinates must fit int32.
constexpr long long kMaxWideBlocks = 1LL << 24;

struct WideLayout {
  size_t table, cache, total;
};

inline WideLayout wide_layout(size_t split_ws_total, int B, int max_blocks) {
  const size_t n = size_t(B) * size_t(max_blocks);
  WideLayout w;
  w.table = align256(split_ws_total);
  w.cache = align256(w.table + n * 4);
  w.total = w.cache + n * kBlock * kRow * 2;
  return w;
}

// Bytes one group of `B` sequences on `P` engines needs: its split-KV
// scratch followed by its widened copy (0 when the copy's block count is out
// of range).
inline size_t fp8_group_bytes(int B, int rows, int max_blocks, int P) {
  if (static_cast<long long>(B) * max_blocks > kMaxWideBlocks) return 0;
  return wide_layout(ws_layout(B, rows, P).total, B, max_blocks).total;
}

// Groups of consecutive sequences, Bg per group (the last one may be short)
// on at most Pg engines, such that every group fits `ws_bytes`: the whole
// batch on P engines when it fits; else fewer engines first (halving), then
// smaller groups (halving, engines back at engines_for(group size)).  Bg = 0
// when not even one sequence on one engine fits.  A group of n sequences runs
// on min(Pg, engines_for(n)) engines.
struct Fp8Plan {
  int Bg, Pg;
};

template <class EnginesFor>
inline Fp8Plan plan_fp8_groups(int B, int rows, int max_blocks, int P, size_t ws_bytes, EnginesFor engines_for) {
  int Bg = B, Pg = P;
  for (;;) {
    const size_t need = fp8_group_bytes(Bg, rows, max_blocks, Pg);
    if (need != 0 && need <= ws_bytes) return Fp8Plan{Bg, Pg};
    if (Pg > 1) {
      Pg = (Pg + 1) / 2;
    } else if (Bg > 1) {
      Bg = (Bg + 1) / 2;
      Pg = engines_for(Bg);
      if (Pg < 1) Pg = 1;
    } else {
      return Fp8Plan{0, 0};
    }
  }
}

}  // namespace mla
