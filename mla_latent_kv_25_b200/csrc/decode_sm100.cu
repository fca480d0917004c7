// Absorbed MLA decode on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One split-KV engine = a cluster of two CTAs on two SMs, split by pipeline
// role because the fp32 output accumulator of 128 heads x 512 latent columns
// fills all 512 TMEM columns of one SM:
//
//   score CTA (rank 0)                         value CTA (rank 1)
//   -----------------                          -----------------
//   w0  TMA: cache rows [64 x 576] -> smem      w0  TMA: latent part [64 x 512] -> smem
//   w1  MMA: S = Q K^T  (A = Q in TMEM,          w1  MMA: O += P V  (A = P, B = V, both
//       B = K tile, N = 64 tokens, K = 576)          smem; V read MN-major from the tile)
//   w4-7 softmax, thread h = head h: online     w2  zero rows past seq_len in the V tile
//       softmax in fp32, P (bf16) and the        w4-7 thread h = head h: rescale O rows when
//       rescale factors to the value CTA             the running max grew, final O / l and
//       by a bulk shared->shared copy                lse (or an fp32 piece of a cut sequence)
//
// Heads are the M = 128 dimension of both contractions (padded with zero
// query rows for H < 128).  The running max is only moved when a block's max
// exceeds it by more than 2^8 (log2 domain), so O is rarely rescaled.
// Every wait is bounded (WaitCtx); a timeout records an error bit and the
// CTA leaves its loops, releases TMEM and exits.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 256;
constexpr int kNK = 2;  // K-tile stages (score CTA)
constexpr int kNV = 2;  // V-tile stages (value CTA)
constexpr int kNP = 2;  // P records in flight
constexpr int kNS = 3;  // S accumulators in TMEM

constexpr uint32_t kChunk = 64 * 128;                  // one [64 rows x 64 bf16] swizzled chunk
constexpr uint32_t kKStage = 9 * kChunk;               // 73728 B: rows [c_kv | k_rope]
constexpr uint32_t kVStage = 8 * kChunk;               // 65536 B: c_kv part only
constexpr uint32_t kPBytes = 128 * 64 * 2;             // P [128 heads x 64 tokens] bf16
constexpr uint32_t kPWarpBytes = 32 * 128;             // one warp's 32 rows of P
constexpr uint32_t kMetaWarp = 400;                    // per warp: alpha[32] m[32] l[32] flag + pad
constexpr uint32_t kMetaBytes = 4 * kMetaWarp;
constexpr float kRescaleThreshold = 8.0f;              // log2 units

// TMEM columns
constexpr uint32_t kQCol = 0;      // score CTA: Q, 576 bf16 = 288 columns
constexpr uint32_t kSCol = 288;    // score CTA: S buffers, 64 columns each
constexpr uint32_t kTmemCols = 512;

struct Barriers {
  uint64_t k_full[kNK], k_empty[kNK];
  uint64_t s_full[kNS], s_empty[kNS];
  uint64_t q_ready, q_free;
  uint64_t p_empty[kNP];
  uint64_t v_full[kNV], v_empty[kNV], v_fixed[kNV];
  uint64_t p_full[kNP];
  uint64_t pv_done, corr_done, o_free;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 1024, "barrier block too large");

// shared-memory offsets from the 1024-aligned base
constexpr uint32_t kRegion = 1024;
__host__ __device__ constexpr uint32_t k_stage_off(int s) { return kRegion + s * kKStage; }
__host__ __device__ constexpr uint32_t p_stage_off(int r) { return kRegion + kNK * kKStage + r * kPBytes; }
__host__ __device__ constexpr uint32_t meta_stage_off(int r) {
  return kRegion + kNK * kKStage + kNP * kPBytes + r * kMetaBytes;
}
__host__ __device__ constexpr uint32_t v_stage_off(int s) { return kRegion + s * kVStage; }
__host__ __device__ constexpr uint32_t p_rec_off(int r) { return kRegion + kNV * kVStage + r * kPBytes; }
__host__ __device__ constexpr uint32_t meta_rec_off(int r) {
  return kRegion + kNV * kVStage + kNP * kPBytes + r * kMetaBytes;
}
constexpr uint32_t kScoreSmem = meta_stage_off(kNP);
constexpr uint32_t kValueSmem = meta_rec_off(kNP);
constexpr uint32_t kSmemBytes = (kScoreSmem > kValueSmem ? kScoreSmem : kValueSmem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(p_stage_off(0) % 1024 == 0 && p_rec_off(0) % 1024 == 0, "swizzle atoms need 1024 B");

constexpr uint32_t kIdescQK = idesc_bf16(128, 64, false, false);   // S[128x64] = Q . K^T
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, false, true);   // O[128x256] += P . V

struct Ctx {
  const DecodeParams* p;
  uint32_t base;        // shared address of the aligned base
  uint8_t* gbase;       // generic pointer to it
  Barriers* bars;
  uint32_t tmem;
  WaitCtx wc;
  int engine;
  int warp, lane;
};

__device__ __forceinline__ uint32_t bar_addr(const Ctx& c, const uint64_t& b) { return smem_u32(&b); }

// all lanes wait; the warp proceeds only if every lane saw the phase complete
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, const WaitCtx& w) {
  bool ok = wait_phase(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// Valid rows of logical block j of segment g (0 for an out-of-range block id);
// *blk receives a block that is safe to load.
__device__ __forceinline__ int block_rows(const DecodeParams& p, const Segment& g, int j,
                                          int* blk) {
  int id = p.block_table[size_t(g.b) * p.max_blocks + j];
  bool ok = id >= 0 && id < p.num_blocks;
  *blk = ok ? id : 0;
  int nv = g.len - j * kBlock;
  nv = nv > kBlock ? kBlock : nv;
  return ok ? nv : 0;
}

// ============================================================ score CTA roles

__device__ void score_tma(const Ctx& c, const CUtensorMap* tmap) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0;
  bool alive = true;
  if (c.lane == 0) prefetch_tmap(tmap);
  while (alive && w.next(g)) {
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      const int s = it % kNK;
      const uint32_t ph = (it / kNK) & 1u;
      if (!warp_wait(bar_addr(c, c.bars->k_empty[s]), ph ^ 1u, c.wc)) {
        alive = false;
        break;
      }
      int blk;
      const int nv = block_rows(p, g, j, &blk);
      if (c.lane == 0) {
        if (nv == 0 && g.len > j * kBlock) atomicOr(p.err, kErrBadBlock);
        const uint32_t full = bar_addr(c, c.bars->k_full[s]);
        mbar_arrive_expect_tx(full, kKStage);
        const uint32_t dst = c.base + k_stage_off(s);
#pragma unroll
        for (int ch = 0; ch < 9; ++ch) tma_load_2d(dst + ch * kChunk, tmap, ch * 64, blk * kBlock, full);
      }
      __syncwarp();
    }
  }
  // wait for the loads this warp issued (bounded) before the CTA may exit
  if (!alive) {
    for (uint32_t k = (it > kNK ? it - kNK : 0); k < it; ++k) {
      const long long t0 = clock64();
      while (!mbar_try_wait(bar_addr(c, c.bars->k_full[k % kNK]), (k / kNK) & 1u) &&
             clock64() - t0 < 2000000000LL) {
      }
    }
  }
}

__device__ void score_mma(const Ctx& c) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0, seg = 0;
  while (w.next(g)) {
    if (!warp_wait(bar_addr(c, c.bars->q_ready), seg & 1u, c.wc)) return;
    tc_fence_after();
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      const int s = it % kNK;
      const int sb = it % kNS;
      if (!warp_wait(bar_addr(c, c.bars->k_full[s]), (it / kNK) & 1u, c.wc)) return;
      if (!warp_wait(bar_addr(c, c.bars->s_empty[sb]), ((it / kNS) & 1u) ^ 1u, c.wc)) return;
      tc_fence_after();
      if (c.lane == 0) {
        const uint32_t d = c.tmem + kSCol + sb * 64;
        const uint32_t kst = c.base + k_stage_off(s);
#pragma unroll 4
        for (int k = 0; k < kRow / 16; ++k) {
          const uint32_t b_addr = kst + (k >> 2) * kChunk + (k & 3) * 32;
          mma_ts(d, c.tmem + kQCol + 8 * k, sw128_desc(b_addr, 16, 1024), kIdescQK, k > 0 ? 1u : 0u);
        }
        mma_commit(bar_addr(c, c.bars->k_empty[s]));
        mma_commit(bar_addr(c, c.bars->s_full[sb]));
      }
      __syncwarp();
    }
    if (c.lane == 0) mma_commit(bar_addr(c, c.bars->q_free));
    __syncwarp();
    ++seg;
  }
}

__device__ void score_softmax(const Ctx& c) {
  const DecodeParams& p = *c.p;
  const int q4 = c.warp - 4;              // TMEM lane quadrant
  const int h = q4 * 32 + c.lane;         // head of this thread
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  const float sl2 = p.softmax_scale * 1.4426950408889634f;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0, seg = 0, pit = 0;
  bool alive = true;
  while (alive && w.next(g)) {
    // ---- this sequence's query row into TMEM (A operand of Q K^T)
    if (seg > 0) {
      if (!warp_wait(bar_addr(c, c.bars->q_free), (seg - 1) & 1u, c.wc)) break;
      tc_fence_after();
    }
    {
      const uint4* src = reinterpret_cast<const uint4*>(p.q + (size_t(g.b) * p.H + h) * kRow);
      const bool live = h < p.H;
#pragma unroll 1
      for (int ch = 0; ch < 9; ++ch) {
        uint32_t r[32];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          uint4 x = live ? __ldg(src + ch * 8 + v) : make_uint4(0, 0, 0, 0);
          r[4 * v] = x.x;
          r[4 * v + 1] = x.y;
          r[4 * v + 2] = x.z;
          r[4 * v + 3] = x.w;
        }
        tmem_st32(c.tmem + lane_off + kQCol + 32 * ch, r);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_addr(c, c.bars->q_ready));
    }
    float m_ref = -INFINITY, l = 0.f;
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it, ++pit) {
      int blk;
      const int nv = block_rows(p, g, j, &blk);
      const int sb = it % kNS;
      if (!warp_wait(bar_addr(c, c.bars->s_full[sb]), (it / kNS) & 1u, c.wc)) {
        alive = false;
        break;
      }
      tc_fence_after();
      uint32_t s0[32], s1[32];
      tmem_ld32(c.tmem + lane_off + kSCol + sb * 64, s0);
      tmem_ld32(c.tmem + lane_off + kSCol + sb * 64 + 32, s1);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar_addr(c, c.bars->s_empty[sb]));

      float x[64];
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        x[t] = t < nv ? __uint_as_float(s0[t]) * sl2 : -INFINITY;
        x[t + 32] = t + 32 < nv ? __uint_as_float(s1[t]) * sl2 : -INFINITY;
      }
      float mx = -INFINITY;
#pragma unroll
      for (int t = 0; t < 64; ++t) mx = fmaxf(mx, x[t]);
      const bool first = (j == g.blk_lo);
      const bool last = (j == g.blk_hi - 1);
      float alpha = 1.f;
      bool resc = false;
      if (first) {
        m_ref = mx;
      } else if (mx > m_ref + kRescaleThreshold) {
        alpha = (m_ref == -INFINITY) ? 0.f : exp2f(m_ref - mx);
        m_ref = mx;
        l *= alpha;
        resc = true;
      }
      uint32_t pk[32];
      float sum = 0.f;
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float e0 = x[2 * t] == -INFINITY ? 0.f : exp2f(x[2 * t] - m_ref);
        const float e1 = x[2 * t + 1] == -INFINITY ? 0.f : exp2f(x[2 * t + 1] - m_ref);
        __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
        const float2 rb = __bfloat1622float2(b2);
        sum += rb.x + rb.y;
        pk[t] = *reinterpret_cast<uint32_t*>(&b2);
      }
      l += sum;

      // ---- ship P and the per-head factors to the value CTA
      const int r = pit % kNP;
      if (!warp_wait(bar_addr(c, c.bars->p_empty[r]), ((pit / kNP) & 1u) ^ 1u, c.wc)) {
        alive = false;
        break;
      }
      uint8_t* prow = c.gbase + p_stage_off(r) + h * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        uint4 v = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(prow + ((ch ^ (h & 7)) << 4)) = v;
      }
      float* meta = reinterpret_cast<float*>(c.gbase + meta_stage_off(r) + q4 * kMetaWarp);
      meta[c.lane] = alpha;
      meta[32 + c.lane] = m_ref;
      meta[64 + c.lane] = l;
      const unsigned any = __any_sync(0xffffffffu, resc);
      if (c.lane == 0) reinterpret_cast<uint32_t*>(meta)[96] = any ? 1u : 0u;
      (void)last;
      fence_proxy_async_smem();
      __syncwarp();
      if (c.lane == 0) {
        const uint32_t full = bar_addr(c, c.bars->p_full[r]);
        mbar_arrive_expect_tx_remote(full, 1, kPWarpBytes + kMetaWarp);
        bulk_copy_to_rank(c.base + p_rec_off(r) + q4 * kPWarpBytes,
                          c.base + p_stage_off(r) + q4 * kPWarpBytes, kPWarpBytes, full, 1);
        bulk_copy_to_rank(c.base + meta_rec_off(r) + q4 * kMetaWarp,
                          c.base + meta_stage_off(r) + q4 * kMetaWarp, kMetaWarp, full, 1);
      }
      __syncwarp();
    }
    ++seg;
  }
  // drain: every record handed to the value CTA has been released, so no
  // remote arrival on this CTA is still pending when it exits
  if (alive) {
    for (uint32_t k = (pit > kNP ? pit - kNP : 0); k < pit; ++k)
      if (!warp_wait(bar_addr(c, c.bars->p_empty[k % kNP]), (k / kNP) & 1u, c.wc)) break;
  }
}

// ============================================================ value CTA roles

__device__ void value_tma(const Ctx& c, const CUtensorMap* tmap) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0;
  bool alive = true;
  if (c.lane == 0) prefetch_tmap(tmap);
  while (alive && w.next(g)) {
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      const int s = it % kNV;
      if (!warp_wait(bar_addr(c, c.bars->v_empty[s]), ((it / kNV) & 1u) ^ 1u, c.wc)) {
        alive = false;
        break;
      }
      int blk;
      block_rows(p, g, j, &blk);
      if (c.lane == 0) {
        const uint32_t full = bar_addr(c, c.bars->v_full[s]);
        mbar_arrive_expect_tx(full, kVStage);
        const uint32_t dst = c.base + v_stage_off(s);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) tma_load_2d(dst + ch * kChunk, tmap, ch * 64, blk * kBlock, full);
      }
      __syncwarp();
    }
  }
  if (!alive) {
    for (uint32_t k = (it > kNV ? it - kNV : 0); k < it; ++k) {
      const long long t0 = clock64();
      while (!mbar_try_wait(bar_addr(c, c.bars->v_full[k % kNV]), (k / kNV) & 1u) &&
             clock64() - t0 < 2000000000LL) {
      }
    }
  }
}

// Rows at or past the valid count of a block are zeroed in the V tile, so that
// whatever the cache holds there (even NaN) contributes exactly 0 * 0.  This
// warp visits every block (arriving on v_fixed even when nothing needs
// zeroing) so that its barrier phases stay in lockstep with the stages.
__device__ void value_fixup(const Ctx& c) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0;
  while (w.next(g)) {
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      int blk;
      const int nv = block_rows(p, g, j, &blk);
      const int s = it % kNV;
      if (!warp_wait(bar_addr(c, c.bars->v_full[s]), (it / kNV) & 1u, c.wc)) return;
      if (nv < kBlock) {
        uint8_t* st = c.gbase + v_stage_off(s);
        const int rows = kBlock - nv;
        for (int idx = c.lane; idx < rows * 8 * 8; idx += 32) {
          const int ch = idx / (rows * 8);
          const int rem = idx % (rows * 8);
          const int row = nv + rem / 8;
          const int q16 = rem % 8;
          *reinterpret_cast<uint4*>(st + ch * kChunk + row * 128 + q16 * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (c.lane == 0) mbar_arrive(bar_addr(c, c.bars->v_fixed[s]));
    }
  }
}

__device__ void value_mma(const Ctx& c) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0, seg = 0, ncorr = 0;
  while (w.next(g)) {
    if (seg > 0) {
      if (!warp_wait(bar_addr(c, c.bars->o_free), (seg - 1) & 1u, c.wc)) return;
      tc_fence_after();
    }
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      int blk;
      const int nv = block_rows(p, g, j, &blk);
      const int s = it % kNV;
      const int r = it % kNP;
      (void)nv;
      if (!warp_wait(bar_addr(c, c.bars->v_full[s]), (it / kNV) & 1u, c.wc)) return;
      if (!warp_wait(bar_addr(c, c.bars->v_fixed[s]), (it / kNV) & 1u, c.wc)) return;
      if (!warp_wait(bar_addr(c, c.bars->p_full[r]), (it / kNP) & 1u, c.wc)) return;
      const bool first = (j == g.blk_lo);
      const uint8_t* meta = c.gbase + meta_rec_off(r);
      uint32_t any = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) any |= reinterpret_cast<const uint32_t*>(meta + q * kMetaWarp)[96];
      if (any && !first) {
        if (!warp_wait(bar_addr(c, c.bars->corr_done), ncorr & 1u, c.wc)) return;
        ++ncorr;
      }
      tc_fence_after();
      if (c.lane == 0) {
        const uint32_t pa = c.base + p_rec_off(r);
        const uint32_t va = c.base + v_stage_off(s);
#pragma unroll
        for (int k = 0; k < kBlock / 16; ++k) {
          const uint64_t adesc = sw128_desc(pa + k * 32, 16, 1024);
#pragma unroll
          for (int n = 0; n < 2; ++n) {
            const uint64_t bdesc = sw128_desc(va + n * 4 * kChunk + k * 2048, kChunk, 1024);
            mma_ss(c.tmem + 256 * n, adesc, bdesc, kIdescPV, (k > 0 || !first) ? 1u : 0u);
          }
        }
        mma_commit(bar_addr(c, c.bars->v_empty[s]));
        mma_commit(bar_addr(c, c.bars->pv_done));
        mma_commit_mc(bar_addr(c, c.bars->p_empty[r]), 0x1);
      }
      __syncwarp();
    }
    ++seg;
  }
}

__device__ void value_epilogue(const Ctx& c) {
  const DecodeParams& p = *c.p;
  const int q4 = c.warp - 4;
  const int h = q4 * 32 + c.lane;
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0;
  while (w.next(g)) {
    float m_fin = -INFINITY, l_fin = 0.f;
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      const int r = it % kNP;
      if (!warp_wait(bar_addr(c, c.bars->p_full[r]), (it / kNP) & 1u, c.wc)) return;
      const uint8_t* meta = c.gbase + meta_rec_off(r);
      const float alpha = reinterpret_cast<const float*>(meta + q4 * kMetaWarp)[c.lane];
      uint32_t any = 0;
#pragma unroll
      for (int q = 0; q < 4; ++q) any |= reinterpret_cast<const uint32_t*>(meta + q * kMetaWarp)[96];
      const bool first = (j == g.blk_lo);
      const bool last = (j == g.blk_hi - 1);
      if (last) {
        m_fin = reinterpret_cast<const float*>(meta + q4 * kMetaWarp)[32 + c.lane];
        l_fin = reinterpret_cast<const float*>(meta + q4 * kMetaWarp)[64 + c.lane];
      }
      __syncwarp();
      if (c.lane == 0) mbar_arrive_remote(bar_addr(c, c.bars->p_empty[r]), 0);
      if (any && !first) {
        // O must hold the previous block's PV before it is rescaled
        if (!warp_wait(bar_addr(c, c.bars->pv_done), (it - 1) & 1u, c.wc)) return;
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < 16; ++ch) {
          uint32_t v[32];
          tmem_ld32(c.tmem + lane_off + 32 * ch, v);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = __float_as_uint(__uint_as_float(v[t]) * alpha);
          tmem_st32(c.tmem + lane_off + 32 * ch, v);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_addr(c, c.bars->corr_done));
      }
      if (last) {
        if (!warp_wait(bar_addr(c, c.bars->pv_done), it & 1u, c.wc)) return;
        tc_fence_after();
        const bool live = h < p.H;
        const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
        const float lse = l_fin > 0.f ? (m_fin + log2f(l_fin)) * 0.6931471805599453f : -INFINITY;
#pragma unroll 1
        for (int ch = 0; ch < 16; ++ch) {
          uint32_t v[32];
          tmem_ld32(c.tmem + lane_off + 32 * ch, v);
          tmem_ld_wait();
          if (!live) continue;
          if (g.slot < 0) {
            uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t(g.b) * p.H + h) * kDc + 32 * ch);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint32_t w4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2 * e]) * inv,
                                                          __uint_as_float(v[8 * q + 2 * e + 1]) * inv);
                w4[e] = *reinterpret_cast<uint32_t*>(&b2);
              }
              dst[q] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          } else {
            float4* dst = reinterpret_cast<float4*>(p.o_part + (size_t(g.slot) * p.H + h) * kDc + 32 * ch);
#pragma unroll
            for (int q = 0; q < 8; ++q)
              dst[q] = make_float4(__uint_as_float(v[4 * q]) * inv, __uint_as_float(v[4 * q + 1]) * inv,
                                   __uint_as_float(v[4 * q + 2]) * inv, __uint_as_float(v[4 * q + 3]) * inv);
          }
        }
        tc_fence_before();
        mbar_arrive(bar_addr(c, c.bars->o_free));
        if (live) {
          if (g.slot < 0)
            p.lse[size_t(g.b) * p.H + h] = lse;
          else
            p.lse_part[size_t(g.slot) * p.H + h] = lse;
        }
        if (h == 0 && g.first_of_seq) p.seq_info[g.b] = seq_info_for(g, w);
      }
    }
  }
}

// ============================================================ kernel

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_sm100_kernel(const __grid_constant__ CUtensorMap tmap, const DecodeParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  Barriers* bars = reinterpret_cast<Barriers*>(gbase);
  const uint32_t rank = cluster_ctarank();
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNK; ++s) {
      mbar_init(smem_u32(&bars->k_full[s]), 1);
      mbar_init(smem_u32(&bars->k_empty[s]), 1);
    }
    for (int s = 0; s < kNS; ++s) {
      mbar_init(smem_u32(&bars->s_full[s]), 1);
      mbar_init(smem_u32(&bars->s_empty[s]), 128);
    }
    mbar_init(smem_u32(&bars->q_ready), 128);
    mbar_init(smem_u32(&bars->q_free), 1);
    for (int r = 0; r < kNP; ++r) {
      mbar_init(smem_u32(&bars->p_empty[r]), 1 + 4);  // PV commit + 4 epilogue warps
      mbar_init(smem_u32(&bars->p_full[r]), 4);       // 4 softmax warps (expect_tx each)
    }
    for (int s = 0; s < kNV; ++s) {
      mbar_init(smem_u32(&bars->v_full[s]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 1);
      mbar_init(smem_u32(&bars->v_fixed[s]), 1);
    }
    mbar_init(smem_u32(&bars->pv_done), 1);
    mbar_init(smem_u32(&bars->corr_done), 128);
    mbar_init(smem_u32(&bars->o_free), 128);
    bars->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();

  Ctx c;
  c.p = &p;
  c.base = base;
  c.gbase = gbase;
  c.bars = bars;
  c.tmem = bars->tmem_base;
  c.wc = WaitCtx{p.spin_limit, p.err, &bars->abort};
  c.engine = blockIdx.x >> 1;
  c.warp = warp;
  c.lane = lane;

  if (rank == 0) {
    if (warp == 0) score_tma(c, &tmap);
    else if (warp == 1) score_mma(c);
    else if (warp >= 4) score_softmax(c);
  } else {
    if (warp == 0) value_tma(c, &tmap);
    else if (warp == 1) value_mma(c);
    else if (warp == 2) value_fixup(c);
    else if (warp >= 4) value_epilogue(c);
  }

  __syncthreads();
  if (bars->abort) {
    // let any asynchronous copy still in flight land before the CTA exits
    if (threadIdx.x == 0) {
      const long long t0 = clock64();
      while (clock64() - t0 < 20000000LL) __nanosleep(1000);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(c.tmem, kTmemCols);
  }
  cluster_sync();
}

}  // namespace

size_t decode_sm100_smem_bytes() { return kSmemBytes; }

cudaError_t launch_decode_sm100(const DecodeParams& p, const CUtensorMap& tmap, cudaStream_t stream) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  decode_sm100_kernel<<<dim3(2 * p.P), kThreads, kSmemBytes, stream>>>(tmap, p);
  return cudaGetLastError();
}

int decode_sm100_max_clusters() {
  if (cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           int(kSmemBytes)) != cudaSuccess)
    return 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_sm100_kernel, &cfg) != cudaSuccess) return 0;
  return n;
}

}  // namespace mla
