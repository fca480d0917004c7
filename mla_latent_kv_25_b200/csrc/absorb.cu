// Query absorption on tcgen05 tensor cores:
//   q_out[b,h,0:512]   = q_nope[b,h,:] . W_UK[h]      (K = 128, fp32 accumulation, one bf16 rounding)
//   q_out[b,h,512:576] = q_rope[b,h,:]                (copied)
//
// One CTA per (head h, tile of 128 batch rows, half of the 512 columns), two
// CTAs per SM.  Per head this is a plain GEMM D[128 x 512] = A[128 x 128] .
// B[128 x 512], each CTA computing one 256-column half:
//   A = q_nope rows of head h (K-major, rows past B read as zeros by TMA),
//   B = the half of W_UK[h] stored [d][c] (c contiguous, so MN-major),
//   D = fp32 in 256 TMEM columns.
// The operands are staged by TMA in two K halves (one barrier each) so the
// MMAs of the first half overlap the second half's load; 8 MMAs of
// 128 x 256 x 16.  The epilogue: each of the 4 warps reads its 32 TMEM lanes
// (= 32 batch rows) and writes bf16 rows.  Splitting the columns doubles the
// CTAs of the launch, so that loads, MMAs and stores of the two halves of a
// head overlap on different SMs instead of running in one CTA in turn.
#include <cuda.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

// Error word of the absorption kernels (the calls have no workspace): bit
// kErrTimeout when a bounded wait gave up.  Read and cleared by
// mla_absorb_get_error.
__device__ uint32_t g_absorb_err;

namespace {

using namespace sm100;

constexpr int kThreads = 128;
constexpr uint32_t kATile = 128 * 128;        // [128 rows x 64 d] bf16, swizzled
constexpr uint32_t kWBox = 64 * 128;          // [64 d x 64 c] bf16
constexpr uint32_t kWChunk = 2 * kWBox;       // [128 d x 64 c]: one 64-column chunk of W_UK[h]
constexpr uint32_t kAOff = 1024;              // after the barrier block
constexpr uint32_t kWOff = kAOff + 2 * kATile;
constexpr int kCols = 256;                    // columns of D per CTA
constexpr int kColChunks = kCols / 64;        // 64-column chunks of W_UK per CTA
constexpr uint32_t kSmem = kWOff + kColChunks * kWChunk + 1024;
static_assert(kSmem <= 232448, "shared memory budget");
constexpr uint32_t kHalfBytes = kATile + kColChunks * kWBox;  // A tile + the W boxes per K half
constexpr uint32_t kIdesc = idesc_bf16(128, 256, false, true);

struct Bars {
  uint64_t full[2];
  uint64_t done;
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(kThreads, 2)
absorb_sm100_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap wmap,
                    const __nv_bfloat16* __restrict__ q_rope, __nv_bfloat16* __restrict__ q_out,
                    int ldq, int B, int H, long long spin_limit) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  Bars* bars = reinterpret_cast<Bars*>(smem_raw + (base - raw));
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * 128;
  const int c0 = blockIdx.z * kCols;            // first output column of this CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars->full[0]), 1);
    mbar_init(smem_u32(&bars->full[1]), 1);
    mbar_init(smem_u32(&bars->done), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars->tmem_base), kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtx wc{spin_limit, &g_absorb_err, &abort_flag};

  if (threadIdx.x == 0) {
    prefetch_tmap(&qmap);
    prefetch_tmap(&wmap);
    for (int kc = 0; kc < 2; ++kc) {
      const uint32_t full = smem_u32(&bars->full[kc]);
      mbar_arrive_expect_tx(full, kHalfBytes);
      // A: d in [64 kc, 64 kc + 64), rows b0..b0+127 of head h
      asm volatile(
          "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
          " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(base + kAOff + kc * kATile),
          "l"(reinterpret_cast<uint64_t>(&qmap)), "r"(64 * kc), "r"(h), "r"(b0), "r"(full)
          : "memory");
      // W_UK[h] rows d in the same half, this CTA's column chunks
      for (int j = 0; j < kColChunks; ++j)
        tma_load_2d(base + kWOff + j * kWChunk + kc * kWBox, &wmap, c0 + 64 * j, h * 128 + 64 * kc, full);
    }
    for (int kc = 0; kc < 2; ++kc) {
      if (!wait_phase(smem_u32(&bars->full[kc]), 0, wc)) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const int k = 4 * kc + kk;  // 16-wide step along d
        const uint64_t a = sw128_desc(base + kAOff + kc * kATile + kk * 32, 16, 1024);
        const uint64_t b = sw128_desc(base + kWOff + k * 2048, kWChunk, 1024);
        mma_ss(tmem, a, b, kIdesc, k > 0 ? 1u : 0u);
      }
    }
    mma_commit(smem_u32(&bars->done));
  }
  __syncwarp();
  const bool ok = warp_wait(smem_u32(&bars->done), 0, wc) && !*static_cast<volatile int*>(&abort_flag);
  tc_fence_after();

  const int row = warp * 32 + lane;
  const int b = b0 + row;
  const bool live = ok && b < B;
  __nv_bfloat16* dst = q_out + (size_t(b) * H + h) * ldq;
#pragma unroll 1
  for (int ch = 0; ch < kCols / 32; ++ch) {
    uint32_t v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 32 * ch, v);
    tmem_ld_wait();
    if (!live) continue;
    uint4* d4 = reinterpret_cast<uint4*>(dst + c0 + 32 * ch);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]),
                                                  __uint_as_float(v[8 * q + 2 * e + 1]));
        w4[e] = *reinterpret_cast<uint32_t*>(&b2);
      }
      d4[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
  if (live && q_rope != nullptr && blockIdx.z == 0) {
    const uint4* src = reinterpret_cast<const uint4*>(q_rope + (size_t(b) * H + h) * kDr);
    uint4* d4 = reinterpret_cast<uint4*>(dst + kDc);
#pragma unroll
    for (int q = 0; q < kDr / 8; ++q) d4[q] = src[q];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kCols);
}

// ---------------------------------------------------------------- output absorption
//   out[b,h,d] = sum_c W_UV[h,d,c] * o_latent[b,h,c]      (d < 128, K = 512)
// One CTA per (head h, 128 batch rows): D[128 x 128] = A[128 x 512] . B^T with
//   A = o_latent rows of head h (K-major; TMA 3-D box {64 c, 1 head, 128 rows},
//       rows past B read as zeros),
//   B = W_UV[h] stored [d][c] (c contiguous: K-major, N = 128 rows),
//   D = fp32 in 128 TMEM columns.
// K streams in four 128-column stages through a ring of two (64 KB each); the
// issuing thread refills a stage once its MMAs have completed.

constexpr uint32_t kOTile = 128 * 128;           // [128 rows x 64 cols] bf16, swizzled
constexpr uint32_t kOStage = 4 * kOTile;         // 2 A tiles + 2 B tiles
constexpr uint32_t kOStageOff = 1024;
constexpr uint32_t kOSmem = kOStageOff + 2 * kOStage + 1024;
static_assert(kOSmem <= 232448, "shared memory budget");
constexpr uint32_t kIdescO = idesc_bf16(128, 128, false, false);

struct OBars {
  uint64_t full[2], empty[2];
  uint64_t done;
  uint32_t tmem_base;
};

__global__ void __launch_bounds__(kThreads, 1)
absorb_o_sm100_kernel(const __grid_constant__ CUtensorMap omap, const __grid_constant__ CUtensorMap wmap,
                      __nv_bfloat16* __restrict__ out, int ldo, int B, int H, long long spin_limit) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  OBars* bars = reinterpret_cast<OBars*>(smem_raw + (base - raw));
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ int abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->done), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&bars->tmem_base), 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const WaitCtx wc{spin_limit, &g_absorb_err, &abort_flag};

  if (threadIdx.x == 0) {
    prefetch_tmap(&omap);
    prefetch_tmap(&wmap);
    auto issue = [&](int k) {  // stage k: latent columns [128 k, 128 k + 128)
      const int s = k & 1;
      const uint32_t full = smem_u32(&bars->full[s]);
      const uint32_t st = base + kOStageOff + s * kOStage;
      mbar_arrive_expect_tx(full, kOStage);
      for (int t = 0; t < 2; ++t) {
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
            " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(st + t * kOTile),
            "l"(reinterpret_cast<uint64_t>(&omap)), "r"(128 * k + 64 * t), "r"(h), "r"(b0), "r"(full)
            : "memory");
        tma_load_2d(st + (2 + t) * kOTile, &wmap, 128 * k + 64 * t, h * 128, full);
      }
    };
    issue(0);
    issue(1);
    for (int k = 0; k < 4; ++k) {
      const int s = k & 1;
      const uint32_t st = base + kOStageOff + s * kOStage;
      if (!wait_phase(smem_u32(&bars->full[s]), (k >> 1) & 1u, wc)) break;
      tc_fence_after();
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(tmem, sw128_desc(st + t * kOTile + kk * 32, 16, 1024),
                 sw128_desc(st + (2 + t) * kOTile + kk * 32, 16, 1024), kIdescO, (k | t | kk) ? 1u : 0u);
      mma_commit(smem_u32(&bars->empty[s]));
      if (k + 2 < 4) {
        if (!wait_phase(smem_u32(&bars->empty[s]), (k >> 1) & 1u, wc)) break;
        issue(k + 2);
      }
    }
    mma_commit(smem_u32(&bars->done));
  }
  __syncwarp();
  const bool ok = warp_wait(smem_u32(&bars->done), 0, wc) && !*static_cast<volatile int*>(&abort_flag);
  tc_fence_after();

  const int b = b0 + warp * 32 + lane;
  const bool live = ok && b < B;
  __nv_bfloat16* dst = out + (size_t(b) * H + h) * ldo;
#pragma unroll 1
  for (int ch = 0; ch < 4; ++ch) {
    uint32_t v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + 32 * ch, v);
    tmem_ld_wait();
    if (!live) continue;
    uint4* d4 = reinterpret_cast<uint4*>(dst + 32 * ch);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t w4[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]),
                                                  __uint_as_float(v[8 * q + 2 * e + 1]));
        w4[e] = *reinterpret_cast<uint32_t*>(&b2);
      }
      d4[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace

cudaError_t launch_absorb_o(const CUtensorMap& omap, const CUtensorMap& wmap, __nv_bfloat16* out,
                            int ldo, int B, int H, long long spin_limit, cudaStream_t stream) {
  // per device, set once (host threads may race to set it; setting it twice is harmless)
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(absorb_o_sm100_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(kOSmem));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  dim3 grid(H, (B + 127) / 128);
  absorb_o_sm100_kernel<<<grid, kThreads, kOSmem, stream>>>(omap, wmap, out, ldo, B, H, spin_limit);
  return cudaGetLastError();
}

cudaError_t launch_absorb_q(const CUtensorMap& qmap, const CUtensorMap& wmap,
                            const __nv_bfloat16* q_rope, __nv_bfloat16* q_out, int ldq, int B,
                            int H, long long spin_limit, cudaStream_t stream) {
  // per device, set once (host threads may race to set it; setting it twice is harmless)
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(absorb_sm100_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmem));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  dim3 grid(H, (B + 127) / 128, kDc / kCols);
  absorb_sm100_kernel<<<grid, kThreads, kSmem, stream>>>(qmap, wmap, q_rope, q_out, ldq, B, H,
                                                         spin_limit);
  return cudaGetLastError();
}

cudaError_t absorb_take_error(uint32_t* bits, cudaStream_t stream) {
  uint32_t* dev = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&dev), g_absorb_err);
  if (e != cudaSuccess) return e;
  if ((e = cudaMemcpyAsync(bits, dev, sizeof(uint32_t), cudaMemcpyDeviceToHost, stream)) != cudaSuccess)
    return e;
  if ((e = cudaMemsetAsync(dev, 0, sizeof(uint32_t), stream)) != cudaSuccess) return e;
  return cudaStreamSynchronize(stream);
}

}  // namespace mla
