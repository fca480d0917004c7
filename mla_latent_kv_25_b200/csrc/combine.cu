// Log-sum-exp merge of split-KV pieces (flash-decoding merge):
//   M = max_i lse_i,  lse = M + log sum_i exp(lse_i - M),
//   out = sum_i exp(lse_i - lse) * o_i
// Each piece o_i is already normalised by its own softmax sum, so the merged
// row equals the softmax over the union of the pieces' tokens.
//
// Two front ends share the row merge:
//   merge_pieces_kernel  - the decode path: pieces live in workspace slots named
//                          by seq_info; also writes length-0 rows and checks
//                          seq_lens.
//   combine_kernel       - the public mla_combine on [B,H,S,512] partials.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kMergeThreads = 128;  // 4 columns per thread

// Merge n pieces of one (b,h) row.  lse_at(i) / o_at(i) give piece i.
// Every thread of the block calls it; thread t owns columns 4t..4t+3.
template <class LseAt, class OAt>
__device__ __forceinline__ void merge_row(int n, LseAt lse_at, OAt o_at, __nv_bfloat16* out_row,
                                          float* lse_out) {
  float M = -INFINITY;
  for (int i = 0; i < n; ++i) M = fmaxf(M, lse_at(i));
  const int c = threadIdx.x * 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float L = -INFINITY;
  if (M != -INFINITY) {
    float sum = 0.f;
    for (int i = 0; i < n; ++i) sum += expf(lse_at(i) - M);
    L = M + logf(sum);
    for (int i = 0; i < n; ++i) {
      float li = lse_at(i);
      if (li == -INFINITY) continue;
      float w = expf(li - L);
      float4 v = *reinterpret_cast<const float4*>(o_at(i) + c);
      acc.x += w * v.x;
      acc.y += w * v.y;
      acc.z += w * v.z;
      acc.w += w * v.w;
    }
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 pk;
  pk.x = *reinterpret_cast<uint32_t*>(&lo);
  pk.y = *reinterpret_cast<uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(out_row + c) = pk;
  if (threadIdx.x == 0) *lse_out = L;
}

// grid (B, ceil(H / heads_per_cta)), 128 threads.
__global__ void __launch_bounds__(kMergeThreads)
merge_pieces_kernel(const int32_t* __restrict__ seq_lens, int max_blocks, int H,
                    const int4* __restrict__ seq_info, const float* __restrict__ lse_part,
                    const float* __restrict__ o_part, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse, uint32_t* __restrict__ err, int heads_per_cta) {
  const int b = blockIdx.x;
  const int h0 = blockIdx.y * heads_per_cta;
  const int h1 = min(H, h0 + heads_per_cta);
  int L = seq_lens[b];
  if (L < 0 || L > max_blocks * kBlock) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, kErrSeqTooLong);
    L = L < 0 ? 0 : max_blocks * kBlock;
  }
  if (L == 0) {
    for (int h = h0; h < h1; ++h) {
      __nv_bfloat16* row = out + (size_t(b) * H + h) * kDc;
      *reinterpret_cast<uint2*>(row + threadIdx.x * 4) = make_uint2(0u, 0u);
      if (threadIdx.x == 0) lse[size_t(b) * H + h] = -INFINITY;
    }
    return;
  }
  const int4 info = seq_info[b];
  if (info.w != kSeqCut) return;  // written directly by its engine
  const int p0 = info.x, p1 = info.y, slot0 = info.z;
  const int n = p1 - p0 + 1;
  for (int h = h0; h < h1; ++h) {
    auto slot_of = [&](int i) { return i == 0 ? slot0 : 2 * (p0 + i); };
    auto lse_at = [&](int i) { return lse_part[size_t(slot_of(i)) * H + h]; };
    auto o_at = [&](int i) { return o_part + (size_t(slot_of(i)) * H + h) * kDc; };
    merge_row(n, lse_at, o_at, out + (size_t(b) * H + h) * kDc, lse + size_t(b) * H + h);
  }
}

// Public combine: o_part [B,H,S,512], lse_part [B,H,S].  grid (B*H), 128 threads.
__global__ void __launch_bounds__(kMergeThreads)
combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, int S,
               __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  const size_t r = blockIdx.x;
  auto lse_at = [&](int i) { return lse_part[r * S + i]; };
  auto o_at = [&](int i) { return o_part + (r * S + i) * kDc; };
  merge_row(S, lse_at, o_at, out + r * kDc, lse + r);
}

}  // namespace

cudaError_t launch_merge_pieces(const int32_t* seq_lens, int B, int max_blocks, int H,
                                const int4* seq_info, const float* lse_part, const float* o_part,
                                __nv_bfloat16* out, float* lse, uint32_t* err,
                                cudaStream_t stream) {
  const int hpc = 8;
  dim3 grid(B, (H + hpc - 1) / hpc);
  merge_pieces_kernel<<<grid, kMergeThreads, 0, stream>>>(seq_lens, max_blocks, H, seq_info,
                                                          lse_part, o_part, out, lse, err, hpc);
  return cudaGetLastError();
}

cudaError_t launch_combine(const float* o_part, const float* lse_part, int B, int H, int S,
                           __nv_bfloat16* out, float* lse, cudaStream_t stream) {
  combine_kernel<<<dim3(unsigned(B) * unsigned(H)), kMergeThreads, 0, stream>>>(o_part, lse_part,
                                                                              S, out, lse);
  return cudaGetLastError();
}

}  // namespace mla
