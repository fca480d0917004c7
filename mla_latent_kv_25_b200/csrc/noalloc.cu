// mla_decode_noalloc: mla_decode with its scratch memory built into the
// library, for callers that cannot allocate device memory themselves.
//
// Who needs it: callers that work inside a fixed memory budget carved out at
// start-up (serving processes that route every later device allocation
// through their own pool and give a library no hook into it), and callers on
// latency-critical paths, where cudaMalloc / cudaFree may synchronise the
// device and take an unbounded time.  Such a caller passes only inputs and
// outputs; the split-KV scratch (error word, per-sequence records, fp32
// partial results of cut sequences) lives in one file-scope device array.
//
// Limits and rules:
//   - The array holds kNoAllocScratchBytes (40 MiB) on every GPU that loads
//     the library, until the process exits.  A request whose scratch need
//     (mla_decode_workspace_bytes(B, H, num_splits)) exceeds it is rejected
//     with MLA_ERR_WORKSPACE_TOO_SMALL and nothing is launched.  At H = 128
//     and the automatic split count of a B200 the need is about 39 MB.
//   - Every call looks up the array's device address on the current device
//     (cudaGetSymbolAddress), so the address stays right after a device reset;
//     make the first call on a device (which loads the module) before any
//     stream capture.
//   - Every call on a device shares the array, which keeps the last call's
//     contents.  Calls whose executions overlap on the GPU (different streams,
//     or host threads racing) race on it; serialise them.
//   - Nothing in the array needs clearing between calls: every value a call
//     reads (per-sequence records, partial results) is written earlier in the
//     same call.  The array starts zeroed when the library is loaded; its
//     error word accumulates device-side error bits of all calls until
//     mla_decode_noalloc_get_error reads and clears it.
//   - An fp8 cache is widened to bf16 rows in the array: the whole batch at
//     once when mla_decode_fp8_workspace_bytes fits in it, else in groups of
//     sequences (as mla_decode does with a smaller workspace).
//   - No device memory is allocated or freed by this entry point.
#include "../../include/mla.h"
#include "common.cuh"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(40) << 20;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device.  Returns
// nullptr on failure.
void* scratch_for_current_device() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess) return nullptr;
  return ptr;
}

}  // namespace

extern "C" mla_status_t mla_decode_noalloc(const void* q, mla_cache_dtype_t cache_dtype,
                                           const void* cache, const void* k_rope,
                                           const float* block_scale, const int32_t* block_table,
                                           const int32_t* seq_lens, int B, int H, int num_blocks,
                                           int max_blocks_per_seq, float softmax_scale, void* out,
                                           float* lse, int num_splits, void* stream) {
  const size_t need = mla_decode_workspace_bytes(B, H, num_splits);
  if (need == 0) return MLA_ERR_INVALID_ARG;
  if (need > kNoAllocScratchBytes) return MLA_ERR_WORKSPACE_TOO_SMALL;
  void* ws = scratch_for_current_device();
  if (ws == nullptr) return MLA_ERR_CUDA;
  return mla_decode(q, cache_dtype, cache, k_rope, block_scale, block_table, seq_lens, B, H,
                    num_blocks, max_blocks_per_seq, softmax_scale, out, lse, ws,
                    kNoAllocScratchBytes, num_splits, stream);
}

extern "C" mla_status_t mla_decode_noalloc_get_error(void* stream, uint32_t* err_bits) {
  if (err_bits == nullptr) return MLA_ERR_INVALID_ARG;
  void* ws = scratch_for_current_device();
  if (ws == nullptr) return MLA_ERR_CUDA;
  return mla_get_device_error(ws, stream, err_bits);
}
