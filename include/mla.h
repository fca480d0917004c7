/*
 * mla.h - C ABI of libmla.so: absorbed Multi-Head Latent Attention decode over
 * a paged latent KV cache, hand-written CUDA for NVIDIA B200 (sm_100a).
 *
 * The method ("Multi-Head Latent Attention: Scaling LLM Serving Throughput via
 * Low-Rank KV Compression", priorstack.com, sections "Empirical Gains" and
 * "Frequently Asked Questions"): every cached token keeps one shared row
 * [c_kv (d_c = 512) | k_rope (d_h^R = 64)]; the key up-projection W_UK is
 * absorbed into the query and W_UV into the output projection, so the decode
 * step attends directly over the latent rows:
 *
 *     q_abs[b,h,:] = q_nope[b,h,:] . W_UK[h]                        (512)
 *     s[b,h,t]     = scale * (q_abs[b,h,:] . c_kv[t] + q_rope[b,h,:] . k_rope[t])
 *     out[b,h,:]   = sum_t softmax_t(s[b,h,:]) c_kv[t]               (512)
 *     lse[b,h]     = log sum_t exp(s[b,h,t])                         (natural log)
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers unless stated otherwise, owned by
 *     the caller.  No call allocates memory (mla_decode_noalloc's scratch is a
 *     file-scope array that exists from load time), and no call synchronises
 *     the stream except the three *_get_error calls, which say so.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *     All work is enqueued on it in order.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns an error status and launches nothing.
 *   - A launch failure returns MLA_ERR_CUDA (cudaGetLastError is consumed).
 *   - Fixed dimensions: d_c = 512, d_h^R = 64, row = 576, 64 tokens per cache
 *     block, 128-wide content query (d_h) for absorption.  H must be a
 *     multiple of 16 in [16, 128].
 *   - bf16 = IEEE binary32 upper half; fp8 = OCP E4M3 (bias 7, max 448, NaN
 *     S.1111.111, no infinities).  Outputs are rounded to nearest even.
 *   - State kept by the library: the wait bound of mla_set_wait_limit
 *     (process-wide), the MLA_SPLITS value (read once per process), per-device
 *     kernel attributes set on first use, the text of each host thread's last
 *     CUDA error (mla_last_error_string) and mla_decode_noalloc's scratch
 *     array (shared by every call on a device).  No other call keeps state
 *     between calls: the caller's workspace carries each decode's scratch and
 *     error word.  Concurrent calls on different streams are safe provided
 *     they use different output and workspace buffers (and, for
 *     mla_decode_noalloc, do not overlap on one device).
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,         /* null pointer, bad size or alignment */
    MLA_ERR_UNSUPPORTED = 2,         /* valid request this build does not handle */
    MLA_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < mla_decode_workspace_bytes(...) */
    MLA_ERR_CUDA = 4,                /* a CUDA runtime/driver call or launch failed */
    MLA_ERR_DEVICE = 5               /* reserved, returned by no call: device-side problems are
                                        MLA_DEVERR_* bits read by the *_get_error calls */
} mla_status_t;

typedef enum {
    MLA_CACHE_BF16 = 0,     /* cache: bf16 [num_blocks, 64, 576] rows [c_kv | k_rope] */
    MLA_CACHE_FP8_E4M3 = 1  /* cache: u8 E4M3 [num_blocks, 64, 512] codes of c_kv / block_scale,
                               k_rope: bf16 [num_blocks, 64, 64], block_scale: f32 [num_blocks] */
} mla_cache_dtype_t;

/* Device-side error bits (read with mla_get_device_error). */
#define MLA_DEVERR_BAD_BLOCK   0x1u  /* a block_table entry needed by seq_lens is < 0 or >= num_blocks */
#define MLA_DEVERR_SEQ_TOO_LONG 0x2u /* seq_lens[b] > 64 * max_blocks_per_seq or < 0 */
#define MLA_DEVERR_TIMEOUT     0x4u  /* a bounded wait inside a kernel gave up; the kernel exited */
#define MLA_DEVERR_BAD_PIECES  0x8u  /* decode: split-KV bookkeeping out of range (internal error);
                                        the affected rows read out = 0, lse = NaN */

/*
 * mla_absorb_q - fold the key up-projection into the query ("Empirical Gains":
 * W^UK is absorbed into the query projection):
 *     q_out[(b*H + h)*ldq + c]       = sum_{d<128} q_nope[b,h,d] * w_uk[h,d,c],  c < 512
 *     q_out[(b*H + h)*ldq + 512 + r] = q_rope[b,h,r],  r < 64   (only if q_rope != NULL)
 * q_nope: bf16 [B,H,128]; w_uk: bf16 [H,128,512]; q_rope: bf16 [B,H,64] or NULL;
 * q_out: bf16 rows of stride ldq elements (ldq >= 512, >= 576 if q_rope != NULL,
 * a multiple of 8; 576 builds the packed [B,H,576] query mla_decode reads).
 * fp32 accumulation (tensor cores), one bf16 rounding.  B >= 1.  All pointers
 * 16-byte aligned; q_nope and w_uk dense in the layouts above.
 */
mla_status_t mla_absorb_q(const void *q_nope, const void *w_uk, const void *q_rope,
                          void *q_out, int ldq, int B, int H, void *stream);

/*
 * mla_absorb_o - the output side of the absorption ("Empirical Gains": W^UV is
 * absorbed into the output projection, so per-head values are never formed):
 *     out[(b*H + h)*ldo + d] = sum_{c<512} w_uv[h,d,c] * o_latent[b,h,c],  d < 128
 * o_latent: bf16 [B,H,512] (e.g. mla_decode's out); w_uv: bf16 [H,128,512];
 * out: bf16 rows of stride ldo elements (ldo >= 128, a multiple of 8).
 * fp32 accumulation (tensor cores), one bf16 rounding.  B >= 1; H in
 * {16,32,...,128}.  All pointers 16-byte aligned; o_latent and w_uv dense.
 */
mla_status_t mla_absorb_o(const void *o_latent, const void *w_uv, void *out, int ldo, int B,
                          int H, void *stream);

/*
 * mla_absorb_get_error - device error bits of the mla_absorb_q / mla_absorb_o launches since
 * the last call (MLA_DEVERR_TIMEOUT when a bounded wait in the kernel gave up;
 * the affected rows are then not written).  Synchronises `stream` and clears
 * the bits.  The error word is one per device and process: absorption calls on
 * different streams (or threads) record into, and this call clears, the same
 * word.  MLA_ERR_INVALID_ARG if err_bits is NULL.
 */
mla_status_t mla_absorb_get_error(void *stream, uint32_t *err_bits);

/*
 * mla_decode_workspace_bytes - bytes of device workspace mla_decode needs for
 * H heads (mla_decode_multi: H = q_len * heads rows, up to 1024, which above
 * 128 need the workspace of one 128-row tile) and `num_splits` split-KV partitions (0 = the automatic count the
 * current device would use).  The workspace holds the device error word and
 * the fp32 partial results of sequences that are cut across partitions.
 * Returns 0 on invalid arguments.
 */
size_t mla_decode_workspace_bytes(int B, int H, int num_splits);

/*
 * mla_decode_fp8_workspace_bytes - workspace bytes that let mla_decode widen
 * the whole batch of an fp8 cache at once: mla_decode_workspace_bytes(B, H, num_splits)
 * rounded up to 256, plus a scratch block table (4 * B * max_blocks_per_seq
 * bytes, rounded up to 256) and a widened bf16 copy of the blocks the batch
 * reads (73,728 bytes per table entry: B * max_blocks_per_seq blocks of
 * 64 x 576 bf16).  Returns 0 on invalid arguments or when
 * B * max_blocks_per_seq exceeds 2^24.
 */
size_t mla_decode_fp8_workspace_bytes(int B, int H, int max_blocks_per_seq, int num_splits);

/*
 * mla_decode - the decode-step attention over the paged latent cache
 * ("Empirical Gains": the cache holds only c^KV and the decoupled RoPE key;
 * "The Memory Wall": the whole cache is streamed from HBM every step).
 *
 * q:           bf16 [B,H,576] = [q_abs | q_rope] per (b,h) (from mla_absorb_q).
 * cache_dtype: MLA_CACHE_BF16 or MLA_CACHE_FP8_E4M3 (see the enum).
 * cache:       bf16 [num_blocks,64,576] or u8 [num_blocks,64,512].
 * k_rope:      fp8 cache only: bf16 [num_blocks,64,64]; must be NULL for bf16.
 * block_scale: fp8 cache only: f32 [num_blocks], c_kv = e4m3(code) * scale;
 *              must be NULL for bf16.
 *              The fp8 cache runs in two kernels: the first writes the rows
 *              a group of sequences reads as bf16
 *              [bf16(e4m3(code) * scale) | k_rope] into the workspace (round
 *              to nearest even: relative error <= 2^-9 per element), the
 *              tensor-core decode then reads them as a bf16 cache.  With
 *              mla_decode_fp8_workspace_bytes(B, H, max_blocks_per_seq,
 *              num_splits) bytes the group is the whole batch; with less,
 *              the call runs the largest groups of consecutive sequences (and
 *              if need be fewer split-KV engines) that fit, one after the
 *              other on `stream`; MLA_ERR_WORKSPACE_TOO_SMALL when not even
 *              one sequence on one engine fits.
 * block_table: int32 [B, max_blocks_per_seq]; logical block j of sequence b is
 *              physical block block_table[b*max_blocks_per_seq + j].  Entries
 *              at j >= ceil(seq_lens[b]/64) are never read (pad with -1).
 * seq_lens:    int32 [B] on the device; 0 <= seq_lens[b] <= 64*max_blocks_per_seq.
 * softmax_scale: multiplies the whole score (both terms) before the softmax.
 * out:         bf16 [B,H,512], the softmax-weighted sum of c_kv per head.
 * lse:         f32 [B,H], natural log of sum_t exp(score); a sequence of
 *              length 0 gives out = 0 and lse = -inf.
 * workspace:   device buffer of >= mla_decode_workspace_bytes(B,H,num_splits)
 *              bytes (fp8 cache: see block_scale), 256-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE; the
 *              library keeps its error word zero except when it records an
 *              error.  One workspace must not be shared by calls that may run
 *              at the same time.
 * num_splits:  number of split-KV partitions (0 = automatic: the environment
 *              variable MLA_SPLITS, read once per process, when it holds an
 *              integer in 1..4096; else chosen from the device's SM count and
 *              B, the same in mla_decode_workspace_bytes).  Results do not
 *              depend on the physical block placement; they may differ in the
 *              last bits between different num_splits.
 *
 * Preconditions checked on the host: non-null pointers, B >= 1, H in
 * {16,32,...,128}, num_blocks >= 1, max_blocks_per_seq >= 1, 16-byte
 * alignment, the fp8-only pointers present exactly for the fp8 cache.
 * Checked on the device (recorded as error bits, the offending rows are
 * skipped): block ids in range, seq_lens in range.  Every internal wait is
 * bounded; on expiry the kernel records MLA_DEVERR_TIMEOUT and exits cleanly.
 * While MLA_DEVERR_TIMEOUT is set in the workspace's error word (it stays set
 * until mla_get_device_error reads it), every row a call writes reads out = 0,
 * lse = NaN, so that no result of an incomplete decode is ever returned.
 */
mla_status_t mla_decode(const void *q, mla_cache_dtype_t cache_dtype, const void *cache,
                        const void *k_rope, const float *block_scale,
                        const int32_t *block_table, const int32_t *seq_lens, int B, int H,
                        int num_blocks, int max_blocks_per_seq, float softmax_scale,
                        void *out, float *lse, void *workspace, size_t workspace_bytes,
                        int num_splits, void *stream);

/*
 * mla_decode_multi - decode q_len query tokens per sequence at once (multi-
 * token prediction / speculative drafts): the q_len * H query rows of a
 * sequence share every cache row they read, so one pass over the cache serves
 * them all.  Token j of sequence b is the (seq_lens[b] - q_len + 1 + j)-th
 * token: it attends to the first seq_lens[b] - (q_len - 1 - j) cached tokens
 * (the drafts' own rows are already in the cache; causal among the drafts).
 * q: bf16 [B, q_len, H, 576]; out: bf16 [B, q_len, H, 512]; lse: f32
 * [B, q_len, H]; bf16 cache only.  q_len * H must be a multiple of 16 and at
 * most 128, or a multiple of 128 up to 1024 with H dividing 128 (e.g. H = 128
 * and q_len = 2..8): such rows are decoded in tiles of 128 rows (whole
 * tokens), one kernel pass over the cache per tile, one tile after the other
 * on `stream`; the tiles read q and write out / lse in place.
 * workspace: mla_decode_workspace_bytes(B, q_len * H, num_splits) bytes.
 * Other arguments and error behaviour as mla_decode; a token that sees no
 * cached token gives out = 0 and lse = -inf.
 */
mla_status_t mla_decode_multi(const void *q, int q_len, const void *cache,
                              const int32_t *block_table, const int32_t *seq_lens, int B, int H,
                              int num_blocks, int max_blocks_per_seq, float softmax_scale,
                              void *out, float *lse, void *workspace, size_t workspace_bytes,
                              int num_splits, void *stream);

/*
 * mla_combine - log-sum-exp merge of S split-KV partial results (the
 * flash-decoding merge that makes split-KV equal the unsplit softmax):
 *     M = max_i lse_part[r,i];  lse[r] = M + log sum_i exp(lse_part[r,i] - M)
 *     out[r,:] = sum_i exp(lse_part[r,i] - lse[r]) * o_part[r,i,:]
 * with r = b*H + h.  o_part: f32 [B,H,S,512] (each piece already normalised by
 * its own softmax sum); lse_part: f32 [B,H,S] (-inf marks an empty piece);
 * out: bf16 [B,H,512]; lse: f32 [B,H].  Rows whose pieces are all -inf give
 * out = 0, lse = -inf.  S >= 1.
 */
mla_status_t mla_combine(const float *o_part, const float *lse_part, int B, int H, int S,
                         void *out, float *lse, void *stream);

/*
 * mla_get_device_error - wait for `stream`, read the MLA_DEVERR_* bits that
 * kernels using `workspace` recorded, and reset them to zero.  *err_bits
 * receives the bits.  Returns MLA_OK, or MLA_ERR_CUDA if the stream or copy
 * failed.  It synchronises the stream (as do mla_absorb_get_error and
 * mla_cache_get_error; no other call does).
 */
mla_status_t mla_get_device_error(void *workspace, void *stream, uint32_t *err_bits);

/*
 * mla_decode_noalloc - mla_decode with its scratch memory built into the
 * library.  The paper has no counterpart: this is a deployment variant for
 * callers that cannot allocate device memory themselves (processes that work
 * inside a fixed budget carved out at start-up and route every later device
 * allocation through their own pool, or latency-critical paths where
 * cudaMalloc/cudaFree may synchronise the device).  Arguments are those of
 * mla_decode without workspace/workspace_bytes; results are the same up to
 * the last bits.
 *
 * Scratch: one file-scope device array of 40 MiB, held on every GPU that
 * loads the library until the process exits.  A request whose scratch need
 * (mla_decode_workspace_bytes(B, H, num_splits)) exceeds 40 MiB returns
 * MLA_ERR_WORKSPACE_TOO_SMALL and launches nothing (at H = 128 the automatic
 * split count of a B200 needs at most about 39 MB).  The first call on a device looks
 * up the array's address on that device; make it before any stream capture.
 * All calls on a device share the array and it keeps the last call's
 * contents: calls that overlap on the GPU race, so serialise them.  Nothing
 * in it needs clearing between calls.  Device-side error bits accumulate in
 * the array's error word; read and clear them with
 * mla_decode_noalloc_get_error (while MLA_DEVERR_TIMEOUT is set there, calls
 * write out = 0, lse = NaN, as mla_decode does).  An fp8 cache is widened in
 * the array: the whole batch when mla_decode_fp8_workspace_bytes(...) fits in
 * the 40 MiB, else in groups of sequences (see mla_decode).  Allocates and
 * frees no device memory.
 */
mla_status_t mla_decode_noalloc(const void *q, mla_cache_dtype_t cache_dtype, const void *cache,
                                const void *k_rope, const float *block_scale,
                                const int32_t *block_table, const int32_t *seq_lens, int B, int H,
                                int num_blocks, int max_blocks_per_seq, float softmax_scale,
                                void *out, float *lse, int num_splits, void *stream);

/*
 * mla_decode_noalloc_get_error - mla_get_device_error for the built-in
 * scratch of mla_decode_noalloc on the current device: waits for `stream`,
 * stores the accumulated MLA_DEVERR_* bits in *err_bits and clears them.
 * MLA_ERR_INVALID_ARG if err_bits is NULL, MLA_ERR_CUDA if the scratch
 * cannot be located or the copy fails.
 */
mla_status_t mla_decode_noalloc_get_error(void *stream, uint32_t *err_bits);

/*
 * mla_cache_append - write the rows of T new tokens into the paged bf16 cache
 * ("Empirical Gains": only c^KV and the decoupled RoPE key are cached; the key
 * is rotated before caching, in fp32 — eeumee.net, FP8/FP32 Mixed Precision):
 *     cache[block_table[b*max_blocks_per_seq + p/64], p%64, :] = [c_kv[t] | RoPE(k_r[t], p)]
 * with b = seq_idx[t], p = pos[t].  RoPE rotates consecutive pairs
 * (x_2i, x_2i+1) by p * 10000^(-2i/64).
 * c_kv: bf16 [T,512] (16-byte aligned); k_r: bf16 [T,64], before rotation;
 * seq_idx, pos: int32 [T] on the device; block_table: int32 [B, max_blocks_per_seq];
 * cache: bf16 [num_blocks,64,576] (16-byte aligned).  Tokens with b or p out
 * of range, or whose block id is out of range, are skipped and recorded as
 * MLA_DEVERR_SEQ_TOO_LONG / MLA_DEVERR_BAD_BLOCK (mla_cache_get_error).  Two
 * tokens must not target the same row.  T = 0 is a no-op.
 */
mla_status_t mla_cache_append(const void *c_kv, const void *k_r, const int32_t *seq_idx,
                              const int32_t *pos, int T, const int32_t *block_table, int B,
                              int max_blocks_per_seq, int num_blocks, void *cache, void *stream);

/*
 * mla_cache_quantize_fp8 - convert n whole blocks of a bf16 cache to the fp8
 * layout mla_decode reads (MLA_CACHE_FP8_E4M3), at the same block ids
 * (eeumee.net, FP8/FP32 Mixed Precision; the per-block scale follows the
 * E4M3 range): for each listed block k,
 *     block_scale[k] = amax_k / 448 (1 if the block's c_kv is all zero),
 *     codes[k, r, c] = E4M3(c_kv[k, r, c] / block_scale[k])  (nearest, saturating),
 *     k_rope[k, r, :] = cache_bf16[k, r, 512:576]  (copied),
 * the divisions in IEEE fp32.  cache_bf16: bf16 [num_blocks,64,576];
 * blocks: int32 [n] on the device; codes: u8 [num_blocks,64,512];
 * k_rope: bf16 [num_blocks,64,64]; block_scale: f32 [num_blocks].  Ids out of
 * range are skipped and recorded as MLA_DEVERR_BAD_BLOCK.  n = 0 is a no-op.
 */
mla_status_t mla_cache_quantize_fp8(const void *cache_bf16, const int32_t *blocks, int n,
                                    int num_blocks, void *codes, void *k_rope, float *block_scale,
                                    void *stream);

/*
 * mla_cache_get_error - device error bits of the cache writers since the last
 * call; synchronises `stream` and clears them.  As for the absorption, the
 * word is one per device and process, shared by calls on every stream.
 * MLA_ERR_INVALID_ARG if err_bits is NULL.
 */
mla_status_t mla_cache_get_error(void *stream, uint32_t *err_bits);

/*
 * mla_set_wait_limit - bound, in SM clock cycles, of every wait inside the
 * decode kernels launched from now on (process-wide; default about two
 * seconds of SM clock; cycles <= 0 restores the default).  Returns the
 * previous bound.  A wait that reaches the bound records MLA_DEVERR_TIMEOUT,
 * makes every role of the kernel leave its loop, lets copies in flight land
 * and exits; the outputs of that launch are then undefined (mla_decode writes
 * them as out = 0, lse = NaN while the bit is set), the context stays
 * usable.  Meant for tests of that failure path and for diagnosis.
 */
long long mla_set_wait_limit(long long cycles);

/* mla_status_string - a static, human-readable name for a status code. */
const char *mla_status_string(mla_status_t status);

/*
 * mla_last_error_string - a static description of the CUDA failure behind the
 * last MLA_ERR_CUDA that a call made on this host thread returned ("no error"
 * before any).  The pointer stays valid until the library is unloaded.
 */
const char *mla_last_error_string(void);

/* mla_num_sms - streaming multiprocessors of the current device (0 on error). */
int mla_num_sms(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
