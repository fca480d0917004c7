// C ABI of libmla.so (declared in include/mla.h): host-side validation,
// workspace layout, choice of the split-KV engine count, and the launches.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdlib.h>

#include <atomic>
#include <mutex>

#include "../../include/mla.h"
#include "common.cuh"
#include "kernels.h"
#include "plan.h"

namespace {

using namespace mla;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Text of the last CUDA failure a call on this host thread returned as
// MLA_ERR_CUDA (mla_last_error_string).
thread_local const char* g_last_error = "no error";

mla_status_t cuda_fail(cudaError_t e) {
  g_last_error = cudaGetErrorString(e);
  return MLA_ERR_CUDA;
}

mla_status_t fail_with(const char* what) {
  g_last_error = what;
  return MLA_ERR_CUDA;
}

mla_status_t status_of(cudaError_t e) { return e == cudaSuccess ? MLA_OK : cuda_fail(e); }

int device_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> g(mu);
  if (dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// Clusters of the tensor-core decode that fit on the device at once.
int device_max_clusters() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  static std::mutex mu;
  static int cache[64] = {0};
  std::lock_guard<std::mutex> g(mu);
  if (dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) cache[dev] = decode_sm100_max_clusters();
  return cache[dev];
}

constexpr int kMaxSplits = 4096;

// MLA_SPLITS=<1..4096> in the environment (read once) replaces the automatic
// engine count; anything else leaves it automatic.
int env_splits() {
  static int value = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    value = 0;
    const char* s = getenv("MLA_SPLITS");
    if (s == nullptr || *s == '\0') return;
    char* end = nullptr;
    const long v = strtol(s, &end, 10);
    if (end != nullptr && *end == '\0' && v >= 1 && v <= kMaxSplits) value = static_cast<int>(v);
  });
  return value;
}

// Engines of the split-KV partition.  By default one per co-resident cluster
// of two SMs; but when the batch is at least three quarters of that and the
// sequences are of similar length, one engine per sequence is faster: no
// sequence is cut (no partial results, no merge) and every engine runs a
// single segment, which outweighs the idle clusters.
int resolve_engines(int num_splits, int B) {
  if (num_splits > 0) return num_splits;
  if (const int env = env_splits(); env > 0) return env;
  int sms = device_sms();
  if (sms < 2) return 0;
  int P = sms / 2;
  int mc = device_max_clusters();
  if (mc > 0 && mc < P) P = mc;
  if (B <= P && 4 * B >= 3 * P) P = B;
  return P;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// bf16 tensor map with 128 B swizzle: dims[0] is the contiguous dimension,
// strides[i] the byte stride of dims[i + 1]; out-of-range reads give zeros.
bool encode_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides, const cuuint32_t* box) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D view [rows, cols] of a row-major bf16 matrix, 64 x 64 box.
bool encode_bf16_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                     uint64_t row_bytes) {
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {64, 64};
  return encode_bf16(map, base, 2, dims, strides, box);
}

constexpr int kMaxBatch = 1 << 20;
constexpr long long kDefaultSpin = 4000000000LL;  // ~2 s of SM clock
std::atomic<long long> g_decode_wait_limit{kDefaultSpin};  // set by mla_set_wait_limit

bool valid_heads(int H) { return H >= 16 && H <= kMaxHeads && H % 16 == 0; }

// Multi-token decode with more than 128 query rows per sequence runs in tiles
// of 128 rows (whole tokens), one decode launch and one cache pass per tile;
// the tiles read q and write out / lse in place (row stride ld_rows).
constexpr int kMaxTiledRows = 8 * kMaxHeads;

bool valid_rows(int rows) {
  return valid_heads(rows) || (rows > kMaxHeads && rows <= kMaxTiledRows && rows % kMaxHeads == 0);
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE: return "MLA_ERR_DEVICE";
  }
  return "MLA_ERR_UNKNOWN";
}

int mla_num_sms(void) { return device_sms(); }

long long mla_set_wait_limit(long long cycles) {
  const long long v = cycles > 0 ? cycles : kDefaultSpin;
  return g_decode_wait_limit.exchange(v);
}

size_t mla_decode_workspace_bytes(int B, int H, int num_splits) {
  if (B < 1 || B > kMaxBatch || !valid_rows(H) || num_splits < 0 || num_splits > kMaxSplits)
    return 0;
  int P = resolve_engines(num_splits, B);
  if (P < 1) return 0;
  return ws_layout(B, H < kMaxHeads ? H : kMaxHeads, P).total;
}

size_t mla_decode_fp8_workspace_bytes(int B, int H, int max_blocks_per_seq, int num_splits) {
  if (max_blocks_per_seq < 1 || max_blocks_per_seq > (1 << 24) || !valid_heads(H)) return 0;
  const size_t base = mla_decode_workspace_bytes(B, H, num_splits);
  if (base == 0) return 0;
  if (static_cast<long long>(B) * max_blocks_per_seq > kMaxWideBlocks) return 0;
  return wide_layout(base, B, max_blocks_per_seq).total;
}

mla_status_t mla_absorb_q(const void* q_nope, const void* w_uk, const void* q_rope, void* q_out,
                          int ldq, int B, int H, void* stream) {
  if (!q_nope || !w_uk || !q_out) return MLA_ERR_INVALID_ARG;
  if (B < 1 || B > kMaxBatch || !valid_heads(H)) return MLA_ERR_INVALID_ARG;
  if (ldq < (q_rope ? kRow : kDc) || ldq % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || !aligned16(w_uk) || !aligned16(q_out) || (q_rope && !aligned16(q_rope)))
    return MLA_ERR_INVALID_ARG;
  // q_nope [B, H, 128] as {d, h, b}: one box = 128 batch rows x 64 d of one head
  CUtensorMap qmap, wmap;
  const cuuint64_t qdims[3] = {cuuint64_t(kNope), cuuint64_t(H), cuuint64_t(B)};
  const cuuint64_t qstr[2] = {cuuint64_t(kNope) * 2, cuuint64_t(H) * kNope * 2};
  const cuuint32_t qbox[3] = {64, 1, 128};
  if (!encode_bf16(&qmap, q_nope, 3, qdims, qstr, qbox)) return fail_with("tensor map encoding failed");
  // W_UK [H, 128, 512] as rows (h, d) x columns c
  if (!encode_bf16_map(&wmap, w_uk, uint64_t(H) * kNope, kDc, kDc * 2))
    return fail_with("tensor map encoding failed");
  cudaError_t e = launch_absorb_q(qmap, wmap, static_cast<const __nv_bfloat16*>(q_rope),
                                  static_cast<__nv_bfloat16*>(q_out), ldq, B, H, kDefaultSpin,
                                  static_cast<cudaStream_t>(stream));
  return status_of(e);
}

mla_status_t mla_absorb_o(const void* o_latent, const void* w_uv, void* out, int ldo, int B, int H,
                          void* stream) {
  if (!o_latent || !w_uv || !out) return MLA_ERR_INVALID_ARG;
  if (B < 1 || B > kMaxBatch || !valid_heads(H)) return MLA_ERR_INVALID_ARG;
  if (ldo < kNope || ldo % 8 != 0) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_latent) || !aligned16(w_uv) || !aligned16(out)) return MLA_ERR_INVALID_ARG;
  CUtensorMap omap, wmap;
  // o_latent [B, H, 512] as {c, h, b}: one box = 128 batch rows x 64 c of one head
  const cuuint64_t odims[3] = {cuuint64_t(kDc), cuuint64_t(H), cuuint64_t(B)};
  const cuuint64_t ostr[2] = {cuuint64_t(kDc) * 2, cuuint64_t(H) * kDc * 2};
  const cuuint32_t obox[3] = {64, 1, 128};
  if (!encode_bf16(&omap, o_latent, 3, odims, ostr, obox)) return fail_with("tensor map encoding failed");
  // W_UV [H, 128, 512] as rows (h, d) x columns c, one box = the 128 rows of a head
  const cuuint64_t wdims[2] = {cuuint64_t(kDc), cuuint64_t(H) * kNope};
  const cuuint64_t wstr[1] = {cuuint64_t(kDc) * 2};
  const cuuint32_t wbox[2] = {64, 128};
  if (!encode_bf16(&wmap, w_uv, 2, wdims, wstr, wbox)) return fail_with("tensor map encoding failed");
  cudaError_t e = launch_absorb_o(omap, wmap, static_cast<__nv_bfloat16*>(out), ldo, B, H,
                                  kDefaultSpin, static_cast<cudaStream_t>(stream));
  return status_of(e);
}

mla_status_t mla_cache_append(const void* c_kv, const void* k_r, const int32_t* seq_idx,
                              const int32_t* pos, int T, const int32_t* block_table, int B,
                              int max_blocks_per_seq, int num_blocks, void* cache, void* stream) {
  if (!c_kv || !k_r || !seq_idx || !pos || !block_table || !cache) return MLA_ERR_INVALID_ARG;
  if (T < 0 || T > kMaxBatch * 64 || B < 1 || B > kMaxBatch) return MLA_ERR_INVALID_ARG;
  if (num_blocks < 1 || max_blocks_per_seq < 1 || max_blocks_per_seq > (1 << 24)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(c_kv) || !aligned16(cache) || (reinterpret_cast<uintptr_t>(k_r) & 3u) ||
      (reinterpret_cast<uintptr_t>(seq_idx) & 3u) || (reinterpret_cast<uintptr_t>(pos) & 3u) ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u))
    return MLA_ERR_INVALID_ARG;
  if (T == 0) return MLA_OK;
  cudaError_t e = launch_cache_append(static_cast<const __nv_bfloat16*>(c_kv),
                                      static_cast<const __nv_bfloat16*>(k_r), seq_idx, pos, T,
                                      block_table, B, max_blocks_per_seq, num_blocks,
                                      static_cast<__nv_bfloat16*>(cache), static_cast<cudaStream_t>(stream));
  return status_of(e);
}

mla_status_t mla_cache_quantize_fp8(const void* cache_bf16, const int32_t* blocks, int n,
                                    int num_blocks, void* codes, void* k_rope, float* block_scale,
                                    void* stream) {
  if (!cache_bf16 || !blocks || !codes || !k_rope || !block_scale) return MLA_ERR_INVALID_ARG;
  if (n < 0 || n > (1 << 24) || num_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (!aligned16(cache_bf16) || !aligned16(codes) || !aligned16(k_rope) ||
      (reinterpret_cast<uintptr_t>(blocks) & 3u) || (reinterpret_cast<uintptr_t>(block_scale) & 3u))
    return MLA_ERR_INVALID_ARG;
  if (n == 0) return MLA_OK;
  cudaError_t e = launch_cache_quantize_fp8(static_cast<const __nv_bfloat16*>(cache_bf16), blocks, n,
                                            num_blocks, static_cast<uint8_t*>(codes),
                                            static_cast<__nv_bfloat16*>(k_rope), block_scale,
                                            static_cast<cudaStream_t>(stream));
  return status_of(e);
}

mla_status_t mla_cache_get_error(void* stream, uint32_t* err_bits) {
  if (!err_bits) return MLA_ERR_INVALID_ARG;
  uint32_t v = 0;
  if (cudaError_t e = cache_take_error(&v, static_cast<cudaStream_t>(stream)); e != cudaSuccess)
    return cuda_fail(e);
  *err_bits = v;
  return MLA_OK;
}

mla_status_t mla_absorb_get_error(void* stream, uint32_t* err_bits) {
  if (!err_bits) return MLA_ERR_INVALID_ARG;
  uint32_t v = 0;
  if (cudaError_t e = absorb_take_error(&v, static_cast<cudaStream_t>(stream)); e != cudaSuccess)
    return cuda_fail(e);
  *err_bits = v;
  return MLA_OK;
}

}  // extern "C"

namespace {

// One decode launch and its merge over a bf16 cache: p's split-KV scratch
// (error word, per-sequence records, partial results) is laid out at the
// start of `workspace` for p.B sequences and p.P engines.
mla_status_t decode_group(DecodeParams p, void* workspace, cudaStream_t st) {
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  const WsLayout ws = ws_layout(p.B, p.H, p.P);
  p.err = reinterpret_cast<uint32_t*>(wsb);
  p.seq_info = reinterpret_cast<int4*>(wsb + ws.seq_info);
  p.lse_part = reinterpret_cast<float*>(wsb + ws.lse_part);
  p.o_part = reinterpret_cast<float*>(wsb + ws.o_part);
  CUtensorMap tmap, qmap;
  if (!encode_bf16_map(&tmap, p.cache, uint64_t(p.num_blocks) * kBlock, kRow, kRow * 2))
    return fail_with("tensor map encoding failed");
  {
    cuuint64_t dims[2] = {uint64_t(kRow), uint64_t(p.B - 1) * uint64_t(p.ld_rows) + uint64_t(p.H)};
    cuuint64_t strides[1] = {uint64_t(kRow) * 2};
    cuuint32_t box[2] = {64, 128};
    if (!encode_bf16(&qmap, p.q, 2, dims, strides, box)) return fail_with("query tensor map encoding failed");
  }
  cudaError_t e = launch_decode_sm100(p, tmap, qmap, st);
  if (e != cudaSuccess) return cuda_fail(e);
  e = launch_merge_pieces(p.seq_lens, p.B, p.max_blocks, p.H, p.ld_rows, p.P, p.seq_info, p.lse_part,
                          p.o_part, p.out, p.lse, p.err, st);
  return status_of(e);
}

// Shared by mla_decode (q_len = 1) and mla_decode_multi: the q_len query
// tokens of a sequence are q_len * H rows of one engine's contraction.
mla_status_t decode_rows(const void* q, int q_len, mla_cache_dtype_t cache_dtype, const void* cache,
                         const void* k_rope, const float* block_scale, const int32_t* block_table,
                         const int32_t* seq_lens, int B, int H, int num_blocks,
                         int max_blocks_per_seq, float softmax_scale, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, int num_splits, void* stream) {
  if (!q || !cache || !block_table || !seq_lens || !out || !lse || !workspace)
    return MLA_ERR_INVALID_ARG;
  if (q_len < 1 || q_len > kMaxTiledRows / 16 || H < 1) return MLA_ERR_INVALID_ARG;
  const int rows = H * q_len;
  if (B < 1 || B > kMaxBatch || !valid_rows(rows)) return MLA_ERR_INVALID_ARG;
  // tiles of 128 rows hold whole tokens: H divides 128
  if (rows > kMaxHeads && (H % 16 != 0 || kMaxHeads % H != 0)) return MLA_ERR_INVALID_ARG;
  if (q_len > 1 && cache_dtype == MLA_CACHE_FP8_E4M3) return MLA_ERR_UNSUPPORTED;
  if (num_blocks < 1 || max_blocks_per_seq < 1 || max_blocks_per_seq > (1 << 24))
    return MLA_ERR_INVALID_ARG;
  if (num_splits < 0 || num_splits > kMaxSplits) return MLA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || isinf(softmax_scale)) return MLA_ERR_INVALID_ARG;
  const bool fp8 = (cache_dtype == MLA_CACHE_FP8_E4M3);
  if (cache_dtype != MLA_CACHE_BF16 && !fp8) return MLA_ERR_INVALID_ARG;
  if (fp8 != (k_rope != nullptr) || fp8 != (block_scale != nullptr)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(cache) || !aligned16(out) || (k_rope && !aligned16(k_rope)) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(block_table) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) != 0 ||
      (block_scale && (reinterpret_cast<uintptr_t>(block_scale) & 3u) != 0))
    return MLA_ERR_INVALID_ARG;
  const int P = resolve_engines(num_splits, B);
  if (P < 1) return fail_with("no streaming multiprocessor count for the current device");
  const int tile = rows < kMaxHeads ? rows : kMaxHeads;
  if (workspace_bytes < ws_layout(B, tile, P).total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  DecodeParams p;
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.cache = cache;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.B = B;
  p.H = tile;
  p.q_len = q_len;
  p.h_per_q = H;
  p.ld_rows = rows;
  p.num_blocks = num_blocks;
  p.max_blocks = max_blocks_per_seq;
  p.softmax_scale = softmax_scale;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.P = P;
  p.spin_limit = g_decode_wait_limit.load();
  if (!fp8) {
    // tile t holds rows [128t, 128t + 128): tokens from t0 = 128t / H on,
    // decoded as the last q_len - t0 tokens of the drafts (so that each row's
    // causal length comes out right); one launch after the other on `stream`
    for (int r0 = 0; r0 < rows; r0 += tile) {
      DecodeParams t = p;
      t.q = p.q + static_cast<size_t>(r0) * kRow;
      t.out = p.out + static_cast<size_t>(r0) * kDc;
      t.lse = p.lse + r0;
      t.q_len = q_len - r0 / H;
      if (mla_status_t s = decode_group(t, workspace, st); s != MLA_OK) return s;
    }
    return MLA_OK;
  }

  // The fp8 cache: each group of sequences is widened to bf16 rows in the
  // workspace, then decoded like a bf16 cache.  One group when the workspace
  // holds the whole batch's widened copy (mla_decode_fp8_workspace_bytes);
  // else the largest groups (and, if need be, fewer split-KV engines) that fit.
  const Fp8Plan plan = plan_fp8_groups(B, rows, max_blocks_per_seq, P, workspace_bytes,
                                       [&](int n) { return resolve_engines(num_splits, n); });
  if (plan.Bg == 0) return MLA_ERR_WORKSPACE_TOO_SMALL;
  const int Bg = plan.Bg, Pg = plan.Pg;
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  for (int b0 = 0; b0 < B; b0 += Bg) {
    const int nb = min(Bg, B - b0);
    const int pg = min(Pg, resolve_engines(num_splits, nb));
    const WideLayout wide = wide_layout(ws_layout(nb, rows, pg).total, nb, max_blocks_per_seq);
    int32_t* wide_table = reinterpret_cast<int32_t*>(wsb + wide.table);
    __nv_bfloat16* wide_cache = reinterpret_cast<__nv_bfloat16*>(wsb + wide.cache);
    const int32_t* table_g = block_table + static_cast<size_t>(b0) * max_blocks_per_seq;
    cudaError_t e = launch_fp8_widen(static_cast<const uint8_t*>(cache),
                                     static_cast<const __nv_bfloat16*>(k_rope), block_scale, table_g,
                                     seq_lens + b0, nb, max_blocks_per_seq, num_blocks, wide_table,
                                     wide_cache, reinterpret_cast<uint32_t*>(wsb), device_sms(), st);
    if (e != cudaSuccess) return cuda_fail(e);
    DecodeParams g = p;
    g.q = p.q + static_cast<size_t>(b0) * rows * kRow;
    g.out = p.out + static_cast<size_t>(b0) * rows * kDc;
    g.lse = p.lse + static_cast<size_t>(b0) * rows;
    g.seq_lens = seq_lens + b0;
    g.B = nb;
    g.P = pg;
    g.cache = wide_cache;
    g.block_table = wide_table;
    g.num_blocks = static_cast<int>(static_cast<long long>(nb) * max_blocks_per_seq);
    if (mla_status_t s = decode_group(g, workspace, st); s != MLA_OK) return s;
  }
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status_t mla_decode(const void* q, mla_cache_dtype_t cache_dtype, const void* cache,
                        const void* k_rope, const float* block_scale, const int32_t* block_table,
                        const int32_t* seq_lens, int B, int H, int num_blocks,
                        int max_blocks_per_seq, float softmax_scale, void* out, float* lse,
                        void* workspace, size_t workspace_bytes, int num_splits, void* stream) {
  return decode_rows(q, 1, cache_dtype, cache, k_rope, block_scale, block_table, seq_lens, B, H,
                     num_blocks, max_blocks_per_seq, softmax_scale, out, lse, workspace,
                     workspace_bytes, num_splits, stream);
}

mla_status_t mla_decode_multi(const void* q, int q_len, const void* cache, const int32_t* block_table,
                              const int32_t* seq_lens, int B, int H, int num_blocks,
                              int max_blocks_per_seq, float softmax_scale, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, int num_splits, void* stream) {
  return decode_rows(q, q_len, MLA_CACHE_BF16, cache, nullptr, nullptr, block_table, seq_lens, B, H,
                     num_blocks, max_blocks_per_seq, softmax_scale, out, lse, workspace,
                     workspace_bytes, num_splits, stream);
}

mla_status_t mla_combine(const float* o_part, const float* lse_part, int B, int H, int S,
                         void* out, float* lse, void* stream) {
  if (!o_part || !lse_part || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (B < 1 || B > kMaxBatch || H < 1 || H > kMaxHeads || S < 1 || S > (1 << 20))
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_part) || !aligned16(out) || (reinterpret_cast<uintptr_t>(lse_part) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return MLA_ERR_INVALID_ARG;
  cudaError_t e = launch_combine(o_part, lse_part, B, H, S, static_cast<__nv_bfloat16*>(out), lse,
                                 static_cast<cudaStream_t>(stream));
  return status_of(e);
}

mla_status_t mla_get_device_error(void* workspace, void* stream, uint32_t* err_bits) {
  if (!workspace || !err_bits) return MLA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  if (cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, st); e != cudaSuccess)
    return cuda_fail(e);
  if (cudaError_t e = cudaStreamSynchronize(st); e != cudaSuccess) return cuda_fail(e);
  *err_bits = v;
  if (v != 0) {
    if (cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof v, st); e != cudaSuccess) return cuda_fail(e);
    if (cudaError_t e = cudaStreamSynchronize(st); e != cudaSuccess) return cuda_fail(e);
  }
  return MLA_OK;
}

const char* mla_last_error_string(void) { return g_last_error; }

}  // extern "C"
