// Writers of the paged latent cache: the steps right before the decode.
//
// cache_append_kernel: one warp per new token t of sequence b at position p
//   writes the row [c_kv | RoPE(k_r, p)] into physical block
//   block_table[b, p / 64], row p % 64 ("Multi-Head Latent Attention: Scaling
//   LLM Serving Throughput via Low-Rank KV Compression", Empirical Gains: only
//   c^KV and the decoupled key k^R are cached; the rotation is applied to k^R
//   before caching, in fp32 — "Multi-Head Latent Attention - Latent KV-Cache
//   (DeepSeek v3)", FP8/FP32 Mixed Precision).  RoPE rotates consecutive pairs
//   (x_2i, x_2i+1) by p * theta_i, theta_i = 10000^(-2i/64); lane i owns pair
//   i.  The angle is formed and reduced modulo 2 pi in double, so long
//   positions keep their accuracy; the rotation itself is fp32.
//
// cache_quantize_fp8_kernel: one CTA per listed block converts the bf16
//   cache block to the fp8 layout: codes = c_kv / scale rounded to E4M3
//   (nearest, saturating), scale = amax / 448 (1 for an all-zero block), both
//   divisions IEEE fp32; the RoPE key columns are copied as bf16.
#include <cuda_fp8.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace mla {

// Error word of the cache writers (the calls have no workspace): bad block
// ids and positions outside the table.  Read and cleared by mla_cache_get_error.
__device__ uint32_t g_cache_err;

namespace {

constexpr int kAppendWarps = 4;

__global__ void __launch_bounds__(32 * kAppendWarps)
cache_append_kernel(const __nv_bfloat16* __restrict__ c_kv, const __nv_bfloat16* __restrict__ k_r,
                    const int32_t* __restrict__ seq_idx, const int32_t* __restrict__ pos, int T,
                    const int32_t* __restrict__ block_table, int B, int max_blocks, int num_blocks,
                    __nv_bfloat16* __restrict__ cache) {
  const int t = blockIdx.x * kAppendWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (t >= T) return;
  const int b = seq_idx[t];
  const int p = pos[t];
  if (b < 0 || b >= B || p < 0 || p >= max_blocks * kBlock) {
    if (lane == 0) atomicOr(&g_cache_err, kErrSeqTooLong);
    return;
  }
  const int blk = block_table[size_t(b) * max_blocks + p / kBlock];
  if (blk < 0 || blk >= num_blocks) {
    if (lane == 0) atomicOr(&g_cache_err, kErrBadBlock);
    return;
  }
  __nv_bfloat16* row = cache + (size_t(blk) * kBlock + p % kBlock) * kRow;
  const uint4* src = reinterpret_cast<const uint4*>(c_kv + size_t(t) * kDc);
  uint4* dst = reinterpret_cast<uint4*>(row);
  dst[lane] = src[lane];
  dst[lane + 32] = src[lane + 32];
  // RoPE pair `lane`
  const __nv_bfloat162 x = reinterpret_cast<const __nv_bfloat162*>(k_r + size_t(t) * kDr)[lane];
  const double theta = pow(10000.0, -2.0 * lane / double(kDr));
  const double kTwoPi = 6.283185307179586476925286766559;
  const double ang = fmod(double(p) * theta, kTwoPi);
  float s, c;
  sincosf(static_cast<float>(ang), &s, &c);
  const float x0 = __bfloat162float(x.x), x1 = __bfloat162float(x.y);
  reinterpret_cast<__nv_bfloat162*>(row + kDc)[lane] =
      __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
}

constexpr int kQuantThreads = 256;

__global__ void __launch_bounds__(kQuantThreads)
cache_quantize_fp8_kernel(const __nv_bfloat16* __restrict__ cache_bf16,
                          const int32_t* __restrict__ blocks, int num_blocks,
                          uint8_t* __restrict__ codes, __nv_bfloat16* __restrict__ k_rope,
                          float* __restrict__ block_scale) {
  __shared__ float red[kQuantThreads / 32];
  const int blk = blocks[blockIdx.x];
  if (blk < 0 || blk >= num_blocks) {
    if (threadIdx.x == 0) atomicOr(&g_cache_err, kErrBadBlock);
    return;
  }
  const __nv_bfloat16* src = cache_bf16 + size_t(blk) * kBlock * kRow;
  // 64 rows x 64 units of 8 latent values
  constexpr int kUnits = kBlock * (kDc / 8);
  float amax = 0.f;
  for (int u = threadIdx.x; u < kUnits; u += kQuantThreads) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + size_t(u / 64) * kRow + (u % 64) * 8);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const float scale = amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f;
  uint8_t* dst = codes + size_t(blk) * kBlock * kDc;
  for (int u = threadIdx.x; u < kUnits; u += kQuantThreads) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + size_t(u / 64) * kRow + (u % 64) * 8);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      const float2 y = make_float2(__fdiv_rn(f.x, scale), __fdiv_rn(f.y, scale));
      const uint32_t pair = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
      w[e >> 1] |= pair << (16 * (e & 1));
    }
    *reinterpret_cast<uint2*>(dst + size_t(u / 64) * kDc + (u % 64) * 8) = make_uint2(w[0], w[1]);
  }
  // RoPE key columns: 64 rows x 8 units of 8 bf16
  for (int u = threadIdx.x; u < kBlock * 8; u += kQuantThreads) {
    const uint4 v = *reinterpret_cast<const uint4*>(src + size_t(u / 8) * kRow + kDc + (u % 8) * 8);
    *reinterpret_cast<uint4*>(k_rope + (size_t(blk) * kBlock + u / 8) * kDr + (u % 8) * 8) = v;
  }
  if (threadIdx.x == 0) block_scale[blk] = scale;
}

}  // namespace

cudaError_t launch_cache_append(const __nv_bfloat16* c_kv, const __nv_bfloat16* k_r,
                                const int32_t* seq_idx, const int32_t* pos, int T,
                                const int32_t* block_table, int B, int max_blocks, int num_blocks,
                                __nv_bfloat16* cache, cudaStream_t stream) {
  const int grid = (T + kAppendWarps - 1) / kAppendWarps;
  cache_append_kernel<<<grid, 32 * kAppendWarps, 0, stream>>>(c_kv, k_r, seq_idx, pos, T, block_table,
                                                              B, max_blocks, num_blocks, cache);
  return cudaGetLastError();
}

cudaError_t launch_cache_quantize_fp8(const __nv_bfloat16* cache_bf16, const int32_t* blocks, int n,
                                      int num_blocks, uint8_t* codes, __nv_bfloat16* k_rope,
                                      float* block_scale, cudaStream_t stream) {
  cache_quantize_fp8_kernel<<<n, kQuantThreads, 0, stream>>>(cache_bf16, blocks, num_blocks, codes,
                                                              k_rope, block_scale);
  return cudaGetLastError();
}

cudaError_t cache_take_error(uint32_t* bits, cudaStream_t stream) {
  uint32_t* dev = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&dev), g_cache_err);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemcpyAsync(bits, dev, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(dev, 0, sizeof(uint32_t), stream)) != cudaSuccess) return e;
  return cudaStreamSynchronize(stream);
}

}  // namespace mla
