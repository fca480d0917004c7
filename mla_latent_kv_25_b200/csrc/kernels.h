// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

struct DecodeParams {
  const __nv_bfloat16* q;          // [B,H,576] (H = rows per sequence)
  const void* cache;               // bf16 [NB,64,576]
  const int32_t* block_table;      // [B,max_blocks]
  const int32_t* seq_lens;         // [B]
  int B, H, num_blocks, max_blocks;
  float softmax_scale;
  __nv_bfloat16* out;              // [B,H,512]
  float* lse;                      // [B,H]
  uint32_t* err;                   // workspace error word
  int4* seq_info;                  // [B]
  float* lse_part;                 // [2P,H]
  float* o_part;                   // [2P,H,512]
  int P;                           // number of split-KV engines
  long long spin_limit;            // bounded-wait limit (clock64 cycles)
  // Multi-token decode: the H rows of a sequence are q_len query tokens of
  // h_per_q heads each (row r = token r / h_per_q); token j sees the
  // sequence without its last q_len - 1 - j tokens.  q_len = 1: plain decode.
  int q_len, h_per_q;
  // Rows between consecutive sequences in q, out and lse (= H, or the whole
  // q_len * heads of a sequence when its rows are decoded in tiles of 128).
  int ld_rows;
};

// Tensor-core decode (bf16 cache): clusters of two CTAs, one engine each.
// `tmap` is a 2-D tiled map over the cache viewed as [num_blocks*64, 576]
// bf16 with a 64 x 64 box and 128-byte swizzle.
// `qmap`: 2-D map over q viewed as [(B - 1) * ld_rows + H, 576] bf16, 64 x 128
// box, 128-byte swizzle (the first query tile of every engine).
cudaError_t launch_decode_sm100(const DecodeParams& p, const CUtensorMap& tmap, const CUtensorMap& qmap,
                                cudaStream_t stream);
size_t decode_sm100_smem_bytes();
int decode_sm100_max_clusters();

cudaError_t launch_merge_pieces(const int32_t* seq_lens, int B, int max_blocks, int H, int ld_rows, int P,
                                const int4* seq_info, const float* lse_part, const float* o_part,
                                __nv_bfloat16* out, float* lse, uint32_t* err,
                                cudaStream_t stream);

cudaError_t launch_combine(const float* o_part, const float* lse_part, int B, int H, int S,
                           __nv_bfloat16* out, float* lse, cudaStream_t stream);

// qmap: 3-D view {d 128, h H, b B} of q_nope with box {64, 1, 128}; wmap: 2-D
// view {c 512, rows H*128} of W_UK with box {64, 64}; both 128 B swizzled.
cudaError_t launch_absorb_q(const CUtensorMap& qmap, const CUtensorMap& wmap,
                            const __nv_bfloat16* q_rope, __nv_bfloat16* q_out, int ldq, int B,
                            int H, long long spin_limit, cudaStream_t stream);
// omap: 3-D view {c 512, h H, b B} of o_latent with box {64, 1, 128}; wmap: 2-D
// view {c 512, rows H*128} of W_UV with box {64, 128}; both 128 B swizzled.
cudaError_t launch_absorb_o(const CUtensorMap& omap, const CUtensorMap& wmap, __nv_bfloat16* out,
                            int ldo, int B, int H, long long spin_limit, cudaStream_t stream);
cudaError_t launch_cache_append(const __nv_bfloat16* c_kv, const __nv_bfloat16* k_r,
                                const int32_t* seq_idx, const int32_t* pos, int T,
                                const int32_t* block_table, int B, int max_blocks, int num_blocks,
                                __nv_bfloat16* cache, cudaStream_t stream);
cudaError_t launch_cache_quantize_fp8(const __nv_bfloat16* cache_bf16, const int32_t* blocks, int n,
                                      int num_blocks, uint8_t* codes, __nv_bfloat16* k_rope,
                                      float* block_scale, cudaStream_t stream);
// Widens the fp8 blocks a batch reads into bf16 rows of a dense scratch cache:
// table entry e = b * max_blocks + j -> wide_table[e] = e and rows
// wide_cache[e, r, :] = [bf16(e4m3(code) * scale) | k_rope] for r below the
// sequence length; wide_table[e] = -1 for unread entries and bad block ids
// (the latter also set kErrBadBlock in *err).
cudaError_t launch_fp8_widen(const uint8_t* codes, const __nv_bfloat16* k_rope,
                             const float* block_scale, const int32_t* block_table,
                             const int32_t* seq_lens, int B, int max_blocks, int num_blocks,
                             int32_t* wide_table, __nv_bfloat16* wide_cache, uint32_t* err,
                             int num_sms, cudaStream_t stream);
// Copies the cache writers' error word to *bits and clears it (synchronises `stream`).
cudaError_t cache_take_error(uint32_t* bits, cudaStream_t stream);
// Copies the absorption kernels' error word to *bits and clears it (synchronises `stream`).
cudaError_t absorb_take_error(uint32_t* bits, cudaStream_t stream);

}  // namespace mla
