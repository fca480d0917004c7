// CUDA-core decode: the same split-KV partition, piece outputs and merge as
// the tensor-core kernel, with plain fp32 FMA arithmetic.  One CTA per
// (engine, group of 16 heads), 256 threads.  Per 64-token block: stage the
// rows in shared memory, 16x64 scores, online softmax (fp32), 16x512 PV.
#include <math.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"

namespace mla {

namespace {

constexpr int kHG = 16;                 // heads per CTA
constexpr int kThreads = 256;
constexpr int kTileStride = kRow / 2 + 1;  // 289 words per row: conflict-free column walks

struct SimtSmem {
  float q[kHG][kRow];
  uint32_t tile[kBlock][kTileStride];   // bf16 pairs
  float p[kHG][kBlock];
  float m[kHG], l[kHG], alpha[kHG];
  float blk_scale;
  Segment seg;
  int have;
};

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ uint32_t fp8x2_to_bf16x2(uint16_t two) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(two), __NV_E4M3);
  __half2 hh = *reinterpret_cast<__half2*>(&h);
  float2 f = __half22float2(hh);
  __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);  // exact: 3 mantissa bits fit
  return *reinterpret_cast<uint32_t*>(&b);
}

template <bool kFp8>
__global__ void __launch_bounds__(kThreads) decode_simt_kernel(DecodeParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SimtSmem& sm = *reinterpret_cast<SimtSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int engine = blockIdx.x;
  const int h0 = blockIdx.y * kHG;

  SegWalker walker;
  if (warp == 0) walker.init(p.seq_lens, p.B, p.max_blocks, p.P, engine);

  for (;;) {
    if (warp == 0) {
      Segment g;
      bool ok = walker.next(g);
      if (lane == 0) {
        sm.have = ok ? 1 : 0;
        if (ok) {
          sm.seg = g;
          if (g.first_of_seq && blockIdx.y == 0) p.seq_info[g.b] = seq_info_for(g, walker);
        }
      }
    }
    __syncthreads();
    if (!sm.have) break;
    const Segment g = sm.seg;
    const int b = g.b;
    // load this sequence's queries
    for (int i = tid; i < kHG * kRow; i += kThreads) {
      int hh = i / kRow, c = i % kRow;
      sm.q[hh][c] = (h0 + hh < p.H) ? __bfloat162float(p.q[(size_t(b) * p.H + h0 + hh) * kRow + c])
                                    : 0.f;
    }
    if (tid < kHG) {
      sm.m[tid] = -INFINITY;
      sm.l[tid] = 0.f;
    }
    float o[kHG][2];
#pragma unroll
    for (int hh = 0; hh < kHG; ++hh) o[hh][0] = o[hh][1] = 0.f;
    __syncthreads();

    const int32_t* trow = p.block_table + size_t(b) * p.max_blocks;
    for (int j = g.blk_lo; j < g.blk_hi; ++j) {
      const int nvalid = min(kBlock, g.len - j * kBlock);
      int blk = trow[j];
      const bool bad = (blk < 0 || blk >= p.num_blocks);
      if (bad) {
        if (tid == 0) atomicOr(p.err, kErrBadBlock);
      }
      // stage the block (rows >= nvalid are not read)
      if (!bad) {
        if (!kFp8) {
          const uint32_t* src = reinterpret_cast<const uint32_t*>(
              static_cast<const __nv_bfloat16*>(p.cache) + size_t(blk) * kBlock * kRow);
          for (int i = tid; i < nvalid * (kRow / 2); i += kThreads) {
            int r = i / (kRow / 2), c = i % (kRow / 2);
            sm.tile[r][c] = src[size_t(r) * (kRow / 2) + c];
          }
        } else {
          const uint16_t* src = reinterpret_cast<const uint16_t*>(
              static_cast<const uint8_t*>(p.cache) + size_t(blk) * kBlock * kDc);
          for (int i = tid; i < nvalid * (kDc / 2); i += kThreads) {
            int r = i / (kDc / 2), c = i % (kDc / 2);
            sm.tile[r][c] = fp8x2_to_bf16x2(src[size_t(r) * (kDc / 2) + c]);
          }
          const uint32_t* kr = reinterpret_cast<const uint32_t*>(p.k_rope + size_t(blk) * kBlock * kDr);
          for (int i = tid; i < nvalid * (kDr / 2); i += kThreads) {
            int r = i / (kDr / 2), c = i % (kDr / 2);
            sm.tile[r][kDc / 2 + c] = kr[size_t(r) * (kDr / 2) + c];
          }
          if (tid == 0) sm.blk_scale = p.block_scale[blk];
        }
      }
      __syncthreads();
      const float bscale = kFp8 ? sm.blk_scale : 1.f;
      // scores: warp w -> heads 2w, 2w+1; lane -> tokens lane, lane+32
      {
        float s[2][2];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int t = 0; t < 2; ++t) s[a][t] = 0.f;
        float sr[2][2];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int t = 0; t < 2; ++t) sr[a][t] = 0.f;
        const int hA = 2 * warp, hB = 2 * warp + 1;
        for (int c2 = 0; c2 < kRow / 2; ++c2) {
          float2 qa = make_float2(sm.q[hA][2 * c2], sm.q[hA][2 * c2 + 1]);
          float2 qb = make_float2(sm.q[hB][2 * c2], sm.q[hB][2 * c2 + 1]);
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            int tok = lane + 32 * t;
            float2 k = unpack_bf16x2(sm.tile[tok][c2]);
            if (c2 < kDc / 2) {
              s[0][t] += qa.x * k.x + qa.y * k.y;
              s[1][t] += qb.x * k.x + qb.y * k.y;
            } else {
              sr[0][t] += qa.x * k.x + qa.y * k.y;
              sr[1][t] += qb.x * k.x + qb.y * k.y;
            }
          }
        }
        // online softmax per head (fp32)
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          const int hh = 2 * warp + a;
          float v[2];
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            int tok = lane + 32 * t;
            v[t] = (tok < nvalid && !bad) ? p.softmax_scale * (bscale * s[a][t] + sr[a][t])
                                          : -INFINITY;
          }
          float mx = fmaxf(v[0], v[1]);
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
          const float m_old = sm.m[hh];
          const float m_new = fmaxf(m_old, mx);
          float e[2], sum = 0.f;
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            e[t] = (v[t] == -INFINITY) ? 0.f : expf(v[t] - m_new);
            sum += e[t];
          }
#pragma unroll
          for (int o2 = 16; o2 > 0; o2 >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o2);
          const float alpha = (m_old == -INFINITY) ? 0.f : expf(m_old - m_new);
          sm.p[hh][lane] = e[0] * bscale;
          sm.p[hh][lane + 32] = e[1] * bscale;
          __syncwarp();
          if (lane == 0) {
            sm.alpha[hh] = (m_new == -INFINITY) ? 1.f : alpha;
            sm.l[hh] = sm.l[hh] * alpha + sum;
            sm.m[hh] = m_new;
          }
        }
      }
      __syncthreads();
      // PV: thread -> latent columns 2*tid, 2*tid+1
#pragma unroll
      for (int hh = 0; hh < kHG; ++hh) {
        float a = sm.alpha[hh];
        o[hh][0] *= a;
        o[hh][1] *= a;
      }
      for (int tok = 0; tok < nvalid && !bad; ++tok) {
        float2 v = unpack_bf16x2(sm.tile[tok][tid]);
#pragma unroll
        for (int hh = 0; hh < kHG; ++hh) {
          float pw = sm.p[hh][tok];
          o[hh][0] += pw * v.x;
          o[hh][1] += pw * v.y;
        }
      }
      __syncthreads();
    }
    // epilogue: normalise, write the row or the piece
#pragma unroll
    for (int hh = 0; hh < kHG; ++hh) {
      const int h = h0 + hh;
      if (h >= p.H) continue;
      const float l = sm.l[hh];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const float lse = (l > 0.f) ? sm.m[hh] + logf(l) : -INFINITY;
      if (g.slot < 0) {
        __nv_bfloat162 v = __floats2bfloat162_rn(o[hh][0] * inv, o[hh][1] * inv);
        *reinterpret_cast<__nv_bfloat162*>(p.out + (size_t(b) * p.H + h) * kDc + 2 * tid) = v;
        if (tid == 0) p.lse[size_t(b) * p.H + h] = lse;
      } else {
        float2 v = make_float2(o[hh][0] * inv, o[hh][1] * inv);
        *reinterpret_cast<float2*>(p.o_part + (size_t(g.slot) * p.H + h) * kDc + 2 * tid) = v;
        if (tid == 0) p.lse_part[size_t(g.slot) * p.H + h] = lse;
      }
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_decode_simt(const DecodeParams& p, bool fp8, cudaStream_t stream) {
  const size_t smem = sizeof(SimtSmem);
  dim3 grid(p.P, (p.H + kHG - 1) / kHG);
  if (fp8) {
    cudaFuncSetAttribute(decode_simt_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(smem));
    decode_simt_kernel<true><<<grid, kThreads, smem, stream>>>(p);
  } else {
    cudaFuncSetAttribute(decode_simt_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         int(smem));
    decode_simt_kernel<false><<<grid, kThreads, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace mla
