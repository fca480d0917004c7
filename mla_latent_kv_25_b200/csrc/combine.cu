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

constexpr int kRowsPerCta = 8;                  // one warp per (b,h) row
constexpr int kMergeThreads = 32 * kRowsPerCta;

// Merge n pieces of one (b,h) row; called by one whole warp, lane l owns
// columns 16l..16l+15.  lse_at(i) / o_at(i) give piece i.
template <class LseAt, class OAt>
__device__ __forceinline__ void merge_row(int n, LseAt lse_at, OAt o_at, __nv_bfloat16* out_row,
                                          float* lse_out, int lane) {
  float M = -INFINITY;
  for (int i = 0; i < n; ++i) M = fmaxf(M, lse_at(i));
  const int c = lane * 16;
  float acc[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) acc[k] = 0.f;
  float L = -INFINITY;
  if (M != -INFINITY) {
    float sum = 0.f;
    for (int i = 0; i < n; ++i) sum += expf(lse_at(i) - M);
    L = M + logf(sum);
    for (int i = 0; i < n; ++i) {
      const float li = lse_at(i);
      if (li == -INFINITY) continue;
      const float w = expf(li - L);
      const float4* src = reinterpret_cast<const float4*>(o_at(i) + c);
      float4 v[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] = src[q];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        acc[4 * q] += w * v[q].x;
        acc[4 * q + 1] += w * v[q].y;
        acc[4 * q + 2] += w * v[q].z;
        acc[4 * q + 3] += w * v[q].w;
      }
    }
  }
  uint32_t pk[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
    pk[k] = *reinterpret_cast<uint32_t*>(&b2);
  }
  uint4* dst = reinterpret_cast<uint4*>(out_row + c);
  dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (lane == 0) *lse_out = L;
}

// grid (B, ceil(H / kRowsPerCta)); warp w merges head blockIdx.y * kRowsPerCta + w.
__global__ void __launch_bounds__(kMergeThreads)
merge_pieces_kernel(const int32_t* __restrict__ seq_lens, int max_blocks, int H, int ld_rows, int P,
                    const int4* __restrict__ seq_info, const float* __restrict__ lse_part,
                    const float* __restrict__ o_part, __nv_bfloat16* __restrict__ out,
                    float* __restrict__ lse, uint32_t* __restrict__ err) {
  // launched with programmatic stream serialization right behind the decode:
  // wait for it to complete (and its writes to be visible) before any read
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31;
  const int h = blockIdx.y * kRowsPerCta + (threadIdx.x >> 5);
  // a decode that gave up (timeout) left seq_info and the pieces incomplete:
  // every row then reads out = 0, lse = NaN instead of stale workspace data
  const bool aborted = (*reinterpret_cast<volatile uint32_t*>(err) & kErrTimeout) != 0;
  int L = seq_lens[b];
  if (L < 0 || L > max_blocks * kBlock) {
    if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(err, kErrSeqTooLong);
    L = L < 0 ? 0 : max_blocks * kBlock;
  }
  if (h >= H) return;
  __nv_bfloat16* row = out + (size_t(b) * ld_rows + h) * kDc;
  auto fill = [&](float lse_value) {
    uint4* dst = reinterpret_cast<uint4*>(row + lane * 16);
    dst[0] = make_uint4(0u, 0u, 0u, 0u);
    dst[1] = make_uint4(0u, 0u, 0u, 0u);
    if (lane == 0) lse[size_t(b) * ld_rows + h] = lse_value;
  };
  if (aborted) {
    fill(NAN);
    return;
  }
  if (L == 0) {
    fill(-INFINITY);
    return;
  }
  const int4 info = seq_info[b];
  if (info.w == kSeqWhole) return;  // written directly by its engine
  const int p0 = info.x, p1 = info.y, slot0 = info.z;
  // the pieces of a cut sequence are engines p0..p1 (slot0 for p0's piece,
  // 2p for the others); anything else is inconsistent bookkeeping
  if (info.w != kSeqCut || p0 < 0 || p1 >= P || p0 > p1 || slot0 < 0 || slot0 >= 2 * P) {
    if (lane == 0) atomicOr(err, kErrBadPieces);
    fill(NAN);
    return;
  }
  const int n = p1 - p0 + 1;
  auto slot_of = [&](int i) { return i == 0 ? slot0 : 2 * (p0 + i); };
  auto lse_at = [&](int i) { return lse_part[size_t(slot_of(i)) * H + h]; };
  auto o_at = [&](int i) { return o_part + (size_t(slot_of(i)) * H + h) * kDc; };
  merge_row(n, lse_at, o_at, row, lse + size_t(b) * ld_rows + h, lane);
}

// Public combine: o_part [B,H,S,512], lse_part [B,H,S].  grid ceil(B*H / kRowsPerCta).
__global__ void __launch_bounds__(kMergeThreads)
combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part, size_t rows,
               int S, __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  const size_t r = size_t(blockIdx.x) * kRowsPerCta + (threadIdx.x >> 5);
  if (r >= rows) return;
  auto lse_at = [&](int i) { return lse_part[r * S + i]; };
  auto o_at = [&](int i) { return o_part + (r * S + i) * kDc; };
  merge_row(S, lse_at, o_at, out + r * kDc, lse + r, threadIdx.x & 31);
}

}  // namespace

cudaError_t launch_merge_pieces(const int32_t* seq_lens, int B, int max_blocks, int H, int ld_rows, int P,
                                const int4* seq_info, const float* lse_part, const float* o_part,
                                __nv_bfloat16* out, float* lse, uint32_t* err,
                                cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(B, (H + kRowsPerCta - 1) / kRowsPerCta);
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_pieces_kernel, seq_lens, max_blocks, H, ld_rows, P, seq_info,
                            lse_part, o_part, out, lse, err);
}

cudaError_t launch_combine(const float* o_part, const float* lse_part, int B, int H, int S,
                           __nv_bfloat16* out, float* lse, cudaStream_t stream) {
  const size_t rows = size_t(B) * size_t(H);
  combine_kernel<<<dim3(unsigned((rows + kRowsPerCta - 1) / kRowsPerCta)), kMergeThreads, 0, stream>>>(
      o_part, lse_part, rows, S, out, lse);
  return cudaGetLastError();
}

}  // namespace mla
