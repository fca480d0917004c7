// Query absorption: q_out[b,h,0:512] = q_nope[b,h,:] . W_UK[h]  (K = 128),
// q_out[b,h,512:576] = q_rope[b,h,:].  One CTA per (head, 16 batch rows);
// thread t owns latent columns 2t, 2t+1; fp32 accumulation, one bf16 rounding.
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kRowsPerCta = 16;
constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
absorb_q_kernel(const __nv_bfloat16* __restrict__ q_nope, const __nv_bfloat16* __restrict__ w_uk,
                const __nv_bfloat16* __restrict__ q_rope, __nv_bfloat16* __restrict__ q_out,
                int ldq, int B, int H) {
  __shared__ float qs[kRowsPerCta][kNope];
  const int h = blockIdx.x;
  const int b0 = blockIdx.y * kRowsPerCta;
  const int nb = min(kRowsPerCta, B - b0);
  const int tid = threadIdx.x;
  for (int i = tid; i < kRowsPerCta * kNope; i += kThreads) {
    int r = i / kNope, d = i % kNope;
    qs[r][d] = r < nb ? __bfloat162float(q_nope[(size_t(b0 + r) * H + h) * kNope + d]) : 0.f;
  }
  __syncthreads();
  float acc[kRowsPerCta][2];
#pragma unroll
  for (int r = 0; r < kRowsPerCta; ++r) acc[r][0] = acc[r][1] = 0.f;
  const __nv_bfloat162* w = reinterpret_cast<const __nv_bfloat162*>(w_uk + size_t(h) * kNope * kDc);
#pragma unroll 4
  for (int d = 0; d < kNope; ++d) {
    float2 wv = __bfloat1622float2(w[size_t(d) * (kDc / 2) + tid]);
#pragma unroll
    for (int r = 0; r < kRowsPerCta; ++r) {
      float a = qs[r][d];
      acc[r][0] += a * wv.x;
      acc[r][1] += a * wv.y;
    }
  }
  for (int r = 0; r < nb; ++r) {
    __nv_bfloat16* dst = q_out + (size_t(b0 + r) * H + h) * ldq;
    reinterpret_cast<__nv_bfloat162*>(dst)[tid] = __floats2bfloat162_rn(acc[r][0], acc[r][1]);
    if (q_rope != nullptr && tid < kDr / 2) {
      const __nv_bfloat162* src =
          reinterpret_cast<const __nv_bfloat162*>(q_rope + (size_t(b0 + r) * H + h) * kDr);
      reinterpret_cast<__nv_bfloat162*>(dst + kDc)[tid] = src[tid];
    }
  }
}

}  // namespace

cudaError_t launch_absorb_q(const __nv_bfloat16* q_nope, const __nv_bfloat16* w_uk,
                            const __nv_bfloat16* q_rope, __nv_bfloat16* q_out, int ldq, int B,
                            int H, cudaStream_t stream) {
  dim3 grid(H, (B + kRowsPerCta - 1) / kRowsPerCta);
  absorb_q_kernel<<<grid, kThreads, 0, stream>>>(q_nope, w_uk, q_rope, q_out, ldq, B, H);
  return cudaGetLastError();
}

}  // namespace mla
