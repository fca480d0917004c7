// Shared device/host definitions of the CUDA path: fixed dimensions, the
// workspace layout, and the split-KV partition of the concatenated block list.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

constexpr int kDc = 512;           // latent width d_c
constexpr int kDr = 64;            // decoupled RoPE key width d_h^R
constexpr int kRow = kDc + kDr;    // one cached row
constexpr int kBlock = 64;         // tokens per cache block
constexpr int kNope = 128;         // content query width d_h (absorption K)
constexpr int kMaxHeads = 128;

constexpr uint32_t kErrBadBlock = 0x1u;
constexpr uint32_t kErrSeqTooLong = 0x2u;
constexpr uint32_t kErrTimeout = 0x4u;
constexpr uint32_t kErrBadPieces = 0x8u;

// ---------------------------------------------------------------------------
// Workspace layout (all offsets 256-byte aligned):
//   [0, 256)            header: uint32 error bits at offset 0; at offsets 4 and 8
//                       where the first timed-out wait gave up (diagnosis)
//   seq_info  int4 [B]  per sequence: (first engine, last engine, slot of the
//                       first engine's piece, kind) written by the decode
//                       kernel, read by the merge kernel
//   lse_part  f32 [2P][H]      lse of each cut piece
//   o_part    f32 [2P][H][512] normalised output of each cut piece
// Engine p owns slots 2p (its first segment) and 2p+1 (a later cut segment).
// ---------------------------------------------------------------------------
struct WsLayout {
  size_t seq_info, lse_part, o_part, total;
};

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

__host__ __device__ inline WsLayout ws_layout(int B, int H, int P) {
  WsLayout w;
  w.seq_info = 256;
  w.lse_part = align256(w.seq_info + size_t(B) * 16);
  w.o_part = align256(w.lse_part + size_t(2 * P) * H * 4);
  w.total = align256(w.o_part + size_t(2 * P) * H * kDc * 4);
  return w;
}

// kind field of seq_info
constexpr int kSeqWhole = 0;   // one engine wrote out/lse directly
constexpr int kSeqCut = 1;     // pieces in slots; the merge kernel combines them

// ---------------------------------------------------------------------------
// Split-KV partition.  The blocks of all sequences are laid end to end
// (sequence-major, NBt in total) and cut into P contiguous, equal ranges:
//   start(p) = floor(p * NBt / P).
// Engine p processes [start(p), start(p+1)).  Only its first and last
// segments can be partial sequences, so at most two pieces per engine.
// ---------------------------------------------------------------------------
__host__ __device__ inline long long range_start(int p, long long NBt, int P) {
  return (static_cast<long long>(p) * NBt) / P;
}

// Engine whose range holds concatenated block x (NBt > 0).
__host__ __device__ inline int engine_of(long long x, long long NBt, int P) {
  return static_cast<int>(((x + 1) * P - 1) / NBt);
}

__device__ __forceinline__ int nblocks_of(int len) { return (len + kBlock - 1) / kBlock; }

// Clamp a sequence length to what the table can address; flags bad values.
__device__ __forceinline__ int checked_len(const int32_t* seq_lens, int b, int max_blocks,
                                           uint32_t* err) {
  int L = seq_lens[b];
  if (L < 0 || L > max_blocks * kBlock) {
    if (err) atomicOr(err, kErrSeqTooLong);
    L = L < 0 ? 0 : max_blocks * kBlock;
  }
  return L;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t v) {
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

}  // namespace mla
