// Widening of an fp8 cache to bf16 rows: the first step of the tensor-core
// decode of an fp8 cache.
//
// The fp8 cache ("Multi-Head Latent Attention - Latent KV-Cache (DeepSeek
// v3)", FP8/FP32 Mixed Precision) stores per 64-token block the E4M3 codes of
// c_kv, one fp32 scale, and the RoPE key in bf16.  The tensor-core decode
// reads bf16 rows [c_kv | k_rope] of 576 values.  For every block a batch
// reads, this kernel writes those rows, c_kv = bf16(e4m3(code) * scale)
// (round to nearest even), into a dense scratch cache held in the workspace:
// logical block j of sequence b lands in scratch block b * max_blocks + j,
// and a scratch block table maps (b, j) to it.  Entries that the decode never
// reads (j at or past the sequence's block count) and bad block ids get -1;
// bad ids also set the bad-block bit, and the decode skips their rows.
//
// One CTA converts one block at a time (grid-stride over the B x max_blocks
// table entries).  A block row is 40 units of 16 bytes read: 32 units of 16
// codes (written as 32 bytes of bf16) and 8 units of 8 RoPE values (copied).
// Each thread loads four units before it stores any, so that every SM keeps
// several loads in flight.  Only rows below the sequence length are written.
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace mla {
namespace {

constexpr int kWidenThreads = 256;
constexpr int kWidenCtasPerSm = 8;                 // 2048 threads: a full SM
constexpr int kCodeUnits = kDc / 16;                // 16 codes per unit
constexpr int kRopeUnits = kDr / 8;                 // 8 bf16 per unit
constexpr int kRowUnits = kCodeUnits + kRopeUnits;  // 40
constexpr int kBatch = 4;                           // units loaded before the stores

// Two codes (low byte first) -> two bf16 of code * scale, packed low first.
__device__ __forceinline__ uint32_t widen_pair(uint32_t pair, float scale) {
  const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(pair & 0xffffu),
                                                   __NV_E4M3);
  const float2 f = __half22float2(__half2(h));
  const __nv_bfloat162 o = __floats2bfloat162_rn(f.x * scale, f.y * scale);
  return *reinterpret_cast<const uint32_t*>(&o);
}

__global__ void __launch_bounds__(kWidenThreads, kWidenCtasPerSm)
fp8_widen_kernel(const uint8_t* __restrict__ codes, const __nv_bfloat16* __restrict__ k_rope,
                 const float* __restrict__ block_scale, const int32_t* __restrict__ block_table,
                 const int32_t* __restrict__ seq_lens, int B, int max_blocks, int num_blocks,
                 int32_t* __restrict__ wide_table, __nv_bfloat16* __restrict__ wide_cache,
                 uint32_t* __restrict__ err) {
  const long long entries = static_cast<long long>(B) * max_blocks;
  for (long long e = blockIdx.x; e < entries; e += gridDim.x) {
    const int b = static_cast<int>(e / max_blocks);
    const int j = static_cast<int>(e % max_blocks);
    // lengths outside [0, 64 * max_blocks] are clamped here and reported by the decode
    int len = seq_lens[b];
    len = len < 0 ? 0 : (len > max_blocks * kBlock ? max_blocks * kBlock : len);
    const int rows = min(kBlock, len - j * kBlock);
    if (rows <= 0) {
      if (threadIdx.x == 0) wide_table[e] = -1;
      continue;
    }
    const int blk = block_table[e];
    if (blk < 0 || blk >= num_blocks) {
      if (threadIdx.x == 0) {
        wide_table[e] = -1;
        atomicOr(err, kErrBadBlock);
      }
      continue;
    }
    if (threadIdx.x == 0) wide_table[e] = static_cast<int32_t>(e);
    const float scale = block_scale[blk];
    const uint8_t* src = codes + static_cast<size_t>(blk) * kBlock * kDc;
    const __nv_bfloat16* rope = k_rope + static_cast<size_t>(blk) * kBlock * kDr;
    __nv_bfloat16* dst = wide_cache + static_cast<size_t>(e) * kBlock * kRow;
    const int units = rows * kRowUnits;
    for (int u0 = threadIdx.x; u0 < units; u0 += kBatch * kWidenThreads) {
      uint4 v[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int u = u0 + k * kWidenThreads;
        if (u < units) {
          const int r = u / kRowUnits, c = u % kRowUnits;
          v[k] = c < kCodeUnits
                     ? *reinterpret_cast<const uint4*>(src + static_cast<size_t>(r) * kDc + c * 16)
                     : *reinterpret_cast<const uint4*>(rope + static_cast<size_t>(r) * kDr +
                                                       (c - kCodeUnits) * 8);
        }
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const int u = u0 + k * kWidenThreads;
        if (u < units) {
          const int r = u / kRowUnits, c = u % kRowUnits;
          __nv_bfloat16* row = dst + static_cast<size_t>(r) * kRow;
          if (c < kCodeUnits) {
            const uint32_t w[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
            uint32_t o[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              o[2 * q] = widen_pair(w[q], scale);
              o[2 * q + 1] = widen_pair(w[q] >> 16, scale);
            }
            uint4* d = reinterpret_cast<uint4*>(row + c * 16);
            d[0] = make_uint4(o[0], o[1], o[2], o[3]);
            d[1] = make_uint4(o[4], o[5], o[6], o[7]);
          } else {
            *reinterpret_cast<uint4*>(row + kDc + (c - kCodeUnits) * 8) = v[k];
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_fp8_widen(const uint8_t* codes, const __nv_bfloat16* k_rope,
                             const float* block_scale, const int32_t* block_table,
                             const int32_t* seq_lens, int B, int max_blocks, int num_blocks,
                             int32_t* wide_table, __nv_bfloat16* wide_cache, uint32_t* err,
                             int num_sms, cudaStream_t stream) {
  const long long entries = static_cast<long long>(B) * max_blocks;
  const long long cap = static_cast<long long>(num_sms > 0 ? num_sms : 148) * kWidenCtasPerSm;
  const int grid = static_cast<int>(entries < cap ? entries : cap);
  fp8_widen_kernel<<<grid, kWidenThreads, 0, stream>>>(codes, k_rope, block_scale, block_table,
                                                       seq_lens, B, max_blocks, num_blocks,
                                                       wide_table, wide_cache, err);
  return cudaGetLastError();
}

}  // namespace mla
