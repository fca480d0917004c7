/*
 * FP64 CPU oracle for the absorbed Multi-Head Latent Attention decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or helper with the CUDA path and must never be used as a
 * fallback for it.
 *
 * What it computes (the plain definition, no blocking, no fusion):
 *
 *   "Multi-Head Latent Attention: Scaling LLM Serving Throughput via Low-Rank
 *   KV Compression" (priorstack.com), section "Empirical Gains": each cached
 *   token holds the compressed latent c^KV (d_c = 512) next to the decoupled
 *   RoPE key k^R (d_h^R = 64); W^UK is absorbed into the query and W^UV into
 *   the output projection, so per-head keys and values are never formed.
 *   With q_abs,h = q_nope,h . W^UK_h, the score of token t for head h is
 *       s_t = scale * ( q_abs,h . c^KV_t + q^R_h . k^R_t )
 *   and the head's latent output is the softmax-weighted sum of c^KV_t,
 *       o_h = sum_t p_t c^KV_t,  p = softmax(s),  lse_h = log sum_t exp(s_t).
 *   The softmax is taken in two passes (max, then exp/sum) in double.
 *
 * Storage formats it reads, widened element by element to double:
 *   bf16: the top 16 bits of an IEEE binary32 (value = bits << 16).
 *   E4M3: OCP 8-bit floating point, 1 sign, 4 exponent (bias 7), 3 mantissa
 *         bits; exponent 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no
 *         infinities.  The fp8 cache stores c^KV / scale[block] per 64-token
 *         block (the FP8/FP32 split of "Multi-Head Latent Attention - Latent
 *         KV-Cache (DeepSeek v3)", eeumee.net, "FP8/FP32 Mixed Precision").
 *
 * Cache layout (paged, 64 tokens per block): logical token t of batch row b
 * lives at physical block block_table[b, t / 64], row t % 64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_DC 512
#define ORC_DR 64
#define ORC_DROW 576
#define ORC_BLOCK 64

enum { ORC_F64 = 0, ORC_BF16 = 1, ORC_E4M3 = 2 };
enum { ORC_OK = 0, ORC_BAD_ARG = 1, ORC_BAD_BLOCK = 2, ORC_NO_MEM = 3 };

double orc_bf16_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double orc_e4m3_to_f64(uint8_t code) {
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

typedef struct {
    int kind;              /* ORC_F64: double [NB,64,576]; ORC_BF16: uint16 [NB,64,576];
                              ORC_E4M3: uint8 [NB,64,512] + k_rope + scale */
    const void *main;
    const uint16_t *k_rope; /* E4M3 only: bf16 bits [NB,64,64] */
    const float *scale;     /* E4M3 only: [NB] */
} orc_cache;

static double cache_elem(const orc_cache *c, int64_t blk, int row, int col) {
    int64_t r = blk * ORC_BLOCK + row;
    switch (c->kind) {
    case ORC_F64:
        return ((const double *)c->main)[r * ORC_DROW + col];
    case ORC_BF16:
        return orc_bf16_to_f64(((const uint16_t *)c->main)[r * ORC_DROW + col]);
    default:
        if (col < ORC_DC)
            return orc_e4m3_to_f64(((const uint8_t *)c->main)[r * ORC_DC + col]) * (double)c->scale[blk];
        return orc_bf16_to_f64(c->k_rope[r * ORC_DR + (col - ORC_DC)]);
    }
}

static double query_elem(int kind, const void *q, int64_t row, int col) {
    if (kind == ORC_F64) return ((const double *)q)[row * ORC_DROW + col];
    return orc_bf16_to_f64(((const uint16_t *)q)[row * ORC_DROW + col]);
}

/* One (b, h) row over logical tokens [t0, t1).  s is scratch of t1 - t0. */
static int decode_one(int q_kind, const void *q, int64_t qrow, const orc_cache *c,
                      const int32_t *table_row, int max_blocks, int num_blocks,
                      int t0, int t1, double scale, double *s, double *o, double *lse) {
    double qv[ORC_DROW];
    for (int i = 0; i < ORC_DROW; ++i) qv[i] = query_elem(q_kind, q, qrow, i);
    for (int i = 0; i < ORC_DC; ++i) o[i] = 0.0;
    if (t1 <= t0) {
        *lse = -INFINITY;
        return ORC_OK;
    }
    /* pass 1: scores (both the latent term and the decoupled RoPE term) */
    for (int t = t0; t < t1; ++t) {
        int j = t / ORC_BLOCK;
        if (j >= max_blocks) return ORC_BAD_BLOCK;
        int32_t blk = table_row[j];
        if (blk < 0 || blk >= num_blocks) return ORC_BAD_BLOCK;
        int r = t % ORC_BLOCK;
        double acc = 0.0;
        for (int i = 0; i < ORC_DC; ++i) acc += qv[i] * cache_elem(c, blk, r, i);
        for (int i = ORC_DC; i < ORC_DROW; ++i) acc += qv[i] * cache_elem(c, blk, r, i);
        s[t - t0] = scale * acc;
    }
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t)
        if (s[t - t0] > m) m = s[t - t0];
    /* pass 2: weights and the weighted sum of the latent rows */
    double l = 0.0;
    for (int t = t0; t < t1; ++t) {
        double w = exp(s[t - t0] - m);
        s[t - t0] = w;
        l += w;
    }
    for (int t = t0; t < t1; ++t) {
        int32_t blk = table_row[t / ORC_BLOCK];
        int r = t % ORC_BLOCK;
        double w = s[t - t0];
        for (int i = 0; i < ORC_DC; ++i) o[i] += w * cache_elem(c, blk, r, i);
    }
    for (int i = 0; i < ORC_DC; ++i) o[i] /= l;
    *lse = m + log(l);
    return ORC_OK;
}

/*
 * Decode a list of units.  units[4*u + 0..3] = (b, h, t0, t1); t1 < 0 means
 * seq_lens[b].  out[u, 512], lse[u].  Returns ORC_OK or an error code.
 */
int orc_decode_units(int q_kind, const void *q, int cache_kind, const void *cache,
                     const uint16_t *k_rope, const float *block_scale,
                     const int32_t *block_table, const int32_t *seq_lens, int B, int H,
                     int num_blocks, int max_blocks, double softmax_scale,
                     const int32_t *units, int n_units, double *out, double *lse,
                     int nthreads) {
    if (!q || !cache || !block_table || !seq_lens || !units || !out || !lse) return ORC_BAD_ARG;
    if (cache_kind == ORC_E4M3 && (!k_rope || !block_scale)) return ORC_BAD_ARG;
    orc_cache c = {cache_kind, cache, k_rope, block_scale};
    int err = ORC_OK;
    int maxlen = 0;
    for (int b = 0; b < B; ++b)
        if (seq_lens[b] > maxlen) maxlen = seq_lens[b];
    for (int u = 0; u < n_units; ++u) {
        int b = units[4 * u], h = units[4 * u + 1];
        if (b < 0 || b >= B || h < 0 || h >= H) return ORC_BAD_ARG;
        if (units[4 * u + 3] > maxlen) maxlen = units[4 * u + 3];
    }
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        if (!s) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
            err = ORC_NO_MEM;
        } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
            for (int u = 0; u < n_units; ++u) {
                int b = units[4 * u], h = units[4 * u + 1];
                int t0 = units[4 * u + 2], t1 = units[4 * u + 3];
                if (t1 < 0) t1 = seq_lens[b];
                if (t0 < 0) t0 = 0;
                int rc = decode_one(q_kind, q, (int64_t)b * H + h, &c,
                                    block_table + (int64_t)b * max_blocks, max_blocks,
                                    num_blocks, t0, t1, softmax_scale, s,
                                    out + (int64_t)u * ORC_DC, lse + u);
                if (rc != ORC_OK) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                    err = rc;
                }
            }
            free(s);
        }
    }
    return err;
}

/*
 * Merge S partial results per row (log-sum-exp merge of split-KV pieces):
 *   M = max_i lse_i, lse = M + log sum_i exp(lse_i - M),
 *   out = sum_i exp(lse_i - lse) o_i.
 * Rows whose partials are all -inf give out = 0 and lse = -inf.
 * o_part[R, S, 512], lse_part[R, S] -> out[R, 512], lse[R].
 */
void orc_combine(const double *o_part, const double *lse_part, int R, int S, double *out,
                 double *lse) {
    for (int r = 0; r < R; ++r) {
        double M = -INFINITY;
        for (int i = 0; i < S; ++i)
            if (lse_part[(int64_t)r * S + i] > M) M = lse_part[(int64_t)r * S + i];
        double *o = out + (int64_t)r * ORC_DC;
        for (int c = 0; c < ORC_DC; ++c) o[c] = 0.0;
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int i = 0; i < S; ++i) sum += exp(lse_part[(int64_t)r * S + i] - M);
        double L = M + log(sum);
        for (int i = 0; i < S; ++i) {
            double li = lse_part[(int64_t)r * S + i];
            if (li == -INFINITY) continue;
            double w = exp(li - L);
            const double *oi = o_part + ((int64_t)r * S + i) * ORC_DC;
            for (int c = 0; c < ORC_DC; ++c) o[c] += w * oi[c];
        }
        lse[r] = L;
    }
}

/*
 * Query absorption, "Empirical Gains" / "Frequently Asked Questions": the key
 * up-projection folds into the query, q_abs[b,h,c] = sum_d q_nope[b,h,d] W_UK[h,d,c].
 * q_nope bf16 [B,H,128], w_uk bf16 [H,128,512] -> out double [B,H,512].
 */
void orc_absorb_q(const uint16_t *q_nope, const uint16_t *w_uk, int B, int H, double *out) {
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            double *o = out + ((int64_t)b * H + h) * ORC_DC;
            for (int c = 0; c < ORC_DC; ++c) o[c] = 0.0;
            for (int d = 0; d < 128; ++d) {
                double a = orc_bf16_to_f64(q_nope[((int64_t)b * H + h) * 128 + d]);
                const uint16_t *w = w_uk + ((int64_t)h * 128 + d) * ORC_DC;
                for (int c = 0; c < ORC_DC; ++c) o[c] += a * orc_bf16_to_f64(w[c]);
            }
        }
}

/*
 * Output absorption ("Empirical Gains": W^UV is absorbed into the output
 * projection, so the head's value vector is never formed per token):
 *     out[b,h,d] = sum_{c<512} W_UV[h,d,c] * o_latent[b,h,c],   d < 128
 * o_latent: bf16 [B,H,512]; w_uv: bf16 [H,128,512]; out: double [B,H,128].
 */
void orc_absorb_o(const uint16_t *o_lat, const uint16_t *w_uv, int B, int H, double *out) {
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            const uint16_t *o = o_lat + ((int64_t)b * H + h) * ORC_DC;
            double *dst = out + ((int64_t)b * H + h) * 128;
            for (int d = 0; d < 128; ++d) {
                const uint16_t *w = w_uv + ((int64_t)h * 128 + d) * ORC_DC;
                double acc = 0.0;
                for (int c = 0; c < ORC_DC; ++c) acc += orc_bf16_to_f64(w[c]) * orc_bf16_to_f64(o[c]);
                dst[d] = acc;
            }
        }
}

int orc_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
