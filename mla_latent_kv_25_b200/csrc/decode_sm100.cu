// Absorbed MLA decode on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One split-KV engine = a cluster of two CTAs on two SMs, split by pipeline
// role because the fp32 output accumulator of 128 heads x 512 latent columns
// fills all 512 TMEM columns of one SM:
//
//   score CTA (rank 0)                           value CTA (rank 1)
//   ------------------                           ------------------
//   w0  TMA: cache rows of three 64-token         w0  TMA: latent part of each block,
//       blocks per pass, one 64-column chunk          half a block (4 chunks) at a time
//       at a time into a ring of [192 x 64] slots     into a ring of [64 x 256] slots
//   w1  MMA: S = Q K^T for 192 tokens at once     w1  MMA: O += P V (A = P, B = V read
//       (N = 192); Q columns 0..255 in TMEM,          MN-major), N = 256 per instruction
//       columns 256..575 in shared memory         w2  zero V rows past seq_len
//   w4-7 softmax, thread h = head h: online       w4-7 thread h = head h: rescale O rows
//       softmax in fp32 per 64-token block;           when the running max grew; final
//       P (bf16) and the rescale factors are         O / l and lse, or an fp32 piece of
//       staged locally                                a cut sequence
//   w2-3 senders: staged records -> value CTA
//       with st.async (overlapping the softmax)
//
// Why N = 192: inside this pipeline an MMA instruction costs roughly 100+
// cycles to issue whatever its N, so 128-token passes ran the QK at half the
// tensor pipe's rate; 192-token passes cut the instructions per block from 18
// to 12.  Two 192-column S buffers leave TMEM room for only half of Q; the
// rest of Q is an SS operand.
// Heads are the M = 128 dimension of both contractions (padded with zero query
// rows for H < 128).  The running max only moves when a block's max exceeds
// it by more than 2^8 (log2 domain), so O is rarely rescaled.  Every wait is
// bounded (WaitCtx); a timeout records an error bit and the CTA leaves its
// loops, releases TMEM and exits.
//
// Barrier discipline: a parity wait can only tell the current phase from the
// one before it, so every barrier here is either observed by its waiters at
// every phase, in order, or used as a strict two-party handshake (q_ready /
// q_free, pv_prev / corr_done, o_ready / o_free).
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
constexpr int kPassBlocks = 3;  // score CTA: blocks per QK pass, so N = 192 per MMA
constexpr int kPassTok = kPassBlocks * 64;
constexpr int kKSlots = 3;      // score CTA: ring of [192 tokens x 64 cols] slots, one column chunk each
constexpr int kVSlots = 5;   // value CTA: ring of [64 tokens x 256 cols] half-block slots
constexpr int kNP = 3;       // P records in flight
constexpr int kNS = 2;       // S accumulators (128 columns each) in TMEM

constexpr uint32_t kChunk = 64 * 128;          // one [64 rows x 64 bf16] swizzled chunk
constexpr uint32_t kKSlot = kPassBlocks * kChunk;  // one column chunk of a pass: [192 rows x 64 bf16]
constexpr uint32_t kVSlot = 4 * kChunk;         // [64 rows x 256 bf16]
constexpr uint32_t kPBytes = 128 * 64 * 2;     // P [128 heads x 64 tokens] bf16
constexpr uint32_t kQTile = 128 * 64 * 2;      // one 64-column chunk of Q [128 heads x 64] bf16
constexpr int kQTmemChunks = 4;                 // Q columns 0..255 live in TMEM (TS operand)
constexpr int kQSmemTiles = 9 - kQTmemChunks;   // columns 256..575 in shared memory (SS operand)
constexpr uint32_t kMetaWarp = 400;            // per warp: alpha[32] m[32] l[32] flag + pad
constexpr uint32_t kMetaBytes = 4 * kMetaWarp;
constexpr float kRescaleThreshold = 8.0f;      // log2 units
constexpr float kLog2e = 1.4426950408889634f;

// TMEM columns of the score CTA: Q columns 0..255 (bf16 pairs: 128 columns),
// then two S buffers of kPassTok fp32 columns each.
constexpr uint32_t kQCol = 0;
constexpr uint32_t kSCol = kQTmemChunks * 32;
static_assert(kSCol + 2 * kPassTok <= 512, "TMEM columns");
constexpr uint32_t kTmemCols = 512;

struct Barriers {
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t s_full[kNS], s_empty[kNS];
  uint64_t q_ready, q_free;
  uint64_t p_empty[kNP];
  uint64_t stage_full[kNP], stage_empty[kNP];
  uint64_t v_full[kVSlots], v_empty[kVSlots], v_fixed[kVSlots];
  uint64_t p_full[kNP];
  uint64_t pv_prev, corr_done, o_ready, o_free;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 1024, "barrier block too large");

// shared-memory offsets from the 1024-aligned base
constexpr uint32_t kRegion = 1024;
__host__ __device__ constexpr uint32_t q_tile_off(int t) { return kRegion + t * kQTile; }
__host__ __device__ constexpr uint32_t k_slot_off(int s) { return kRegion + kQSmemTiles * kQTile + s * kKSlot; }
// score CTA staging of the P records and factors before the bulk copy
__host__ __device__ constexpr uint32_t p_stage_off(int r) { return k_slot_off(kKSlots) + r * kPBytes; }
__host__ __device__ constexpr uint32_t meta_stage_off(int r) {
  return k_slot_off(kKSlots) + kNP * kPBytes + r * kMetaBytes;
}
__host__ __device__ constexpr uint32_t v_slot_off(int s) { return kRegion + s * kVSlot; }
__host__ __device__ constexpr uint32_t p_rec_off(int r) { return kRegion + kVSlots * kVSlot + r * kPBytes; }
__host__ __device__ constexpr uint32_t meta_rec_off(int r) {
  return kRegion + kVSlots * kVSlot + kNP * kPBytes + r * kMetaBytes;
}
constexpr uint32_t kScoreSmem = meta_stage_off(kNP);
constexpr uint32_t kValueSmem = meta_rec_off(kNP);
constexpr uint32_t kSmemBytes = (kScoreSmem > kValueSmem ? kScoreSmem : kValueSmem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(k_slot_off(0) % 1024 == 0 && p_rec_off(0) % 1024 == 0 && p_stage_off(0) % 1024 == 0,
              "swizzle atoms need 1024 B");

constexpr uint32_t kIdescQK = idesc_bf16(128, kPassTok, false, false);  // S[128 x 192] = Q . K^T
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, false, true);   // O[128x256] += P . V

struct Ctx {
  const DecodeParams* p;
  uint32_t base;   // shared address of the aligned base
  uint8_t* gbase;  // generic pointer to it
  Barriers* bars;
  uint32_t tmem;
  WaitCtx wc;
  int engine;
  int warp, lane;
};

__device__ __forceinline__ uint32_t bar_addr(const uint64_t& b) { return smem_u32(&b); }

// Physical block ids of one sequence, fetched 32 at a time by the whole warp
// (one global load per 32 blocks instead of one per block).
struct BlockCursor {
  const int32_t* row;
  int nblk;
  int base;
  int cached;

  __device__ void reset(const DecodeParams& p, const Segment& g) {
    row = p.block_table + size_t(g.b) * p.max_blocks;
    nblk = nblocks_of(g.len);
    base = -64;
    cached = -1;
  }
  // id of logical block j (warp-uniform j < nblk)
  __device__ int id(int j, int lane) {
    if (j < base || j >= base + 32) {
      base = j;
      cached = (j + lane < nblk) ? row[j + lane] : -1;
    }
    return __shfl_sync(0xffffffffu, cached, j - base);
  }
};

// Valid rows of logical block j of segment g (0 for an out-of-range block id);
// *blk receives a block that is safe to load.
__device__ __forceinline__ int block_rows(const DecodeParams& p, const Segment& g, BlockCursor& cur,
                                          int j, int lane, int* blk) {
  const int id = cur.id(j, lane);
  const bool ok = id >= 0 && id < p.num_blocks;
  *blk = ok ? id : 0;
  int nv = g.len - j * kBlock;
  nv = nv > kBlock ? kBlock : nv;
  return ok ? nv : 0;
}

// ============================================================ score CTA roles

// kPassBlocks consecutive blocks of a segment form one pass (fewer at the end
// of the segment); each pass streams its 9 column chunks through the slot
// ring, one chunk of all the pass's blocks per slot.
__device__ void score_tma(const Ctx& c, const CUtensorMap* tmap) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  BlockCursor cur;
  uint32_t cit = 0;
  bool alive = true;
  if (c.lane == 0) prefetch_tmap(tmap);
  while (alive && w.next(g)) {
    cur.reset(p, g);
    for (int j = g.blk_lo; alive && j < g.blk_hi; j += kPassBlocks) {
      const int nb = min(kPassBlocks, g.blk_hi - j);
      int blk[kPassBlocks];
#pragma unroll
      for (int k = 0; k < kPassBlocks; ++k) {
        blk[k] = 0;
        if (k < nb) {
          // every block of the segment holds at least one token: 0 rows = bad id
          if (block_rows(p, g, cur, j + k, c.lane, &blk[k]) == 0 && c.lane == 0)
            atomicOr(p.err, kErrBadBlock);
        }
      }
      for (int ch = 0; ch < 9; ++ch, ++cit) {
        const int s = cit % kKSlots;
        if (!warp_wait(bar_addr(c.bars->k_empty[s]), ((cit / kKSlots) & 1u) ^ 1u, c.wc)) {
          alive = false;
          break;
        }
        if (c.lane == 0) {
          const uint32_t full = bar_addr(c.bars->k_full[s]);
          mbar_arrive_expect_tx(full, static_cast<uint32_t>(nb) * kChunk);
          const uint32_t dst = c.base + k_slot_off(s);
#pragma unroll
          for (int k = 0; k < kPassBlocks; ++k)
            if (k < nb) tma_load_2d(dst + k * kChunk, tmap, ch * 64, blk[k] * kBlock, full);
        }
        __syncwarp();
      }
    }
  }
  // wait (bounded) for the loads this warp issued before the CTA may exit
  if (!alive) {
    for (uint32_t k = (cit > kKSlots ? cit - kKSlots : 0); k < cit; ++k) {
      const long long t0 = clock64();
      while (!mbar_test_wait(bar_addr(c.bars->k_full[k % kKSlots]), (k / kKSlots) & 1u) &&
             clock64() - t0 < 2000000000LL) {
      }
    }
  }
}

// The whole warp walks the segments (the walker uses warp collectives), but
// each segment's issue loop runs in one single-thread region of lane 0:
// issuing a slot's MMAs from a lane-0 branch that the warp enters and leaves
// every slot measured about twice the cycles per MMA of a single-thread loop.
__device__ bool score_mma_segment(const Ctx& c, const Segment& g, uint32_t seg, uint32_t& cit,
                                  uint32_t& pit) {
  const uint32_t tmem = c.tmem;
  const uint32_t qs = c.base + q_tile_off(0);
  const uint32_t kbase = c.base + k_slot_off(0);
  Barriers* bars = c.bars;
  if (!wait_phase(bar_addr(bars->q_ready), seg & 1u, c.wc)) return false;
  tc_fence_after();
  for (int j = g.blk_lo; j < g.blk_hi; j += kPassBlocks, ++pit) {
    const int sb = pit % kNS;
    if (!wait_phase(bar_addr(bars->s_empty[sb]), ((pit / kNS) & 1u) ^ 1u, c.wc)) return false;
    const uint32_t d = tmem + kSCol + sb * kPassTok;
    for (int ch = 0; ch < 9; ++ch, ++cit) {
      const int s = cit % kKSlots;
      if (!wait_phase(bar_addr(bars->k_full[s]), (cit / kKSlots) & 1u, c.wc)) return false;
      tc_fence_after();
      const uint32_t tile = kbase + s * kKSlot;
      if (ch < kQTmemChunks) {
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(d, tmem + kQCol + 32 * ch + 8 * kk, sw128_desc(tile + kk * 32, 16, 1024), kIdescQK,
                 (ch | kk) ? 1u : 0u);
      } else {
        const uint32_t qt = qs + (ch - kQTmemChunks) * kQTile;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss(d, sw128_desc(qt + kk * 32, 16, 1024), sw128_desc(tile + kk * 32, 16, 1024), kIdescQK, 1u);
      }
      mma_commit(bar_addr(bars->k_empty[s]));
    }
    mma_commit(bar_addr(bars->s_full[sb]));
  }
  mma_commit(bar_addr(bars->q_free));
  return true;
}

__device__ void score_mma(const Ctx& c) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t cit = 0, pit = 0, seg = 0;
  while (w.next(g)) {
    int ok = 1;
    if (c.lane == 0) ok = score_mma_segment(c, g, seg, cit, pit) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ok, 0)) return;
    ++seg;
  }
}

// Query row of sequence b for head h: columns 0..255 into TMEM lane h as 128
// packed columns (the TS operand of the first four column chunks), columns
// 256..575 into five swizzled [128 x 64] K-major tiles in shared memory (the
// SS operand of the last five).
__device__ __forceinline__ void load_q_rows(const DecodeParams& p, int b, int h, uint32_t taddr,
                                            uint8_t* qtiles) {
  const bool live = h < p.H;
  const uint4* src = reinterpret_cast<const uint4*>(p.q + (size_t(b) * p.H + (live ? h : 0)) * kRow);
  const uint4 z = make_uint4(0, 0, 0, 0);
  const uint32_t swz = static_cast<uint32_t>(h & 7);
#pragma unroll
  for (int ch = 0; ch < 9; ++ch) {
    uint4 v8[8];
#pragma unroll
    for (int v = 0; v < 8; ++v) v8[v] = live ? __ldg(src + ch * 8 + v) : z;
    if (ch < kQTmemChunks) {
      uint32_t r[32];
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        r[4 * v] = v8[v].x;
        r[4 * v + 1] = v8[v].y;
        r[4 * v + 2] = v8[v].z;
        r[4 * v + 3] = v8[v].w;
      }
      tmem_st32(taddr + 32 * ch, r);
    } else {
      uint8_t* row = qtiles + (ch - kQTmemChunks) * kQTile + h * 128;
#pragma unroll
      for (int v = 0; v < 8; ++v)
        *reinterpret_cast<uint4*>(row + ((static_cast<uint32_t>(v) ^ swz) << 4)) = v8[v];
    }
  }
}
__device__ __forceinline__ void prefetch_q_rows_l2(const DecodeParams& p, int b, int h) {
  if (h >= p.H) return;
  const char* src = reinterpret_cast<const char*>(p.q + (size_t(b) * p.H + h) * kRow);
#pragma unroll
  for (int i = 0; i < 9; ++i) asm volatile("prefetch.global.L2 [%0];" ::"l"(src + 128 * i));
}

struct SoftmaxState {
  float m_ref, l;
};

// Online softmax of one 64-token block (raw scores in sv) and its hand-off to
// the value CTA.  Returns false if a wait gave up.
__device__ __forceinline__ bool softmax_block(const Ctx& c, const uint32_t (&sv)[64], int nv, bool first,
                                              float sl2, bool pos, SoftmaxState& st, uint32_t it,
                                              int h, int q4) {
  // block max of the scaled scores: max of s * sg with sg = sign(scale), so a
  // negative scale needs no second code path; rows at or past nv are masked
  const float sg = pos ? 1.f : -1.f;
  float mr = -INFINITY;
#pragma unroll
  for (int t = 0; t < 64; ++t) mr = fmaxf(mr, t < nv ? __uint_as_float(sv[t]) * sg : -INFINITY);
  const float mx = nv > 0 ? mr * sg * sl2 : -INFINITY;
  float alpha = 1.f;
  bool resc = false;
  if (first) {
    st.m_ref = mx;
  } else if (mx > st.m_ref + kRescaleThreshold) {
    alpha = (st.m_ref == -INFINITY) ? 0.f : ex2_approx(st.m_ref - mx);
    st.m_ref = mx;
    st.l *= alpha;
    resc = true;
  }
  const float neg_m = st.m_ref == -INFINITY ? 0.f : -st.m_ref;
  uint32_t pk[32];
  float sum = 0.f;
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    float e0 = ex2_approx(fmaf(__uint_as_float(sv[2 * t]), sl2, neg_m));
    float e1 = ex2_approx(fmaf(__uint_as_float(sv[2 * t + 1]), sl2, neg_m));
    e0 = 2 * t < nv ? e0 : 0.f;
    e1 = 2 * t + 1 < nv ? e1 : 0.f;
    sum += e0 + e1;
    __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
    pk[t] = *reinterpret_cast<uint32_t*>(&b2);
  }
  st.l += sum;

  // P row and the per-head factors into this CTA's staging record r; the
  // sender warps move it to the value CTA
  const int r = it % kNP;
  if (!warp_wait(bar_addr(c.bars->stage_empty[r]), ((it / kNP) & 1u) ^ 1u, c.wc)) return false;
  uint8_t* prow = c.gbase + p_stage_off(r) + h * 128;
  const uint32_t swz = static_cast<uint32_t>(h & 7);
#pragma unroll
  for (int ch = 0; ch < 8; ++ch)
    *reinterpret_cast<uint4*>(prow + ((static_cast<uint32_t>(ch) ^ swz) << 4)) =
        make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
  float* meta = reinterpret_cast<float*>(c.gbase + meta_stage_off(r) + q4 * kMetaWarp);
  meta[c.lane] = alpha;
  meta[32 + c.lane] = st.m_ref;
  meta[64 + c.lane] = st.l;
  const unsigned any = __any_sync(0xffffffffu, resc);
  if (c.lane == 0) reinterpret_cast<uint32_t*>(meta)[96] = any ? 1u : 0u;
  mbar_arrive(bar_addr(c.bars->stage_full[r]));
  return true;
}

__device__ void score_softmax(const Ctx& c) {
  const DecodeParams& p = *c.p;
  const int q4 = c.warp - 4;              // TMEM lane quadrant
  const int h = q4 * 32 + c.lane;         // head of this thread
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  const float sl2 = p.softmax_scale * kLog2e;
  const bool pos = sl2 >= 0.f;
  uint8_t* qtiles = c.gbase + q_tile_off(0);
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  BlockCursor cur;
  uint32_t it = 0, pit = 0, seg = 0;
  bool alive = true;
  while (alive && w.next(g)) {
    cur.reset(p, g);
    if (seg > 0) {
      if (!warp_wait(bar_addr(c.bars->q_free), (seg - 1) & 1u, c.wc)) break;
      tc_fence_after();
    }
    load_q_rows(p, g.b, h, c.tmem + lane_off + kQCol, qtiles);
    fence_proxy_async_smem();
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(bar_addr(c.bars->q_ready));
    if (w.b < w.B && w.pre < w.e) prefetch_q_rows_l2(p, w.b, h);  // next segment's query

    SoftmaxState st{-INFINITY, 0.f};
    // multi-token decode: this row's query token sees the sequence without
    // its last `short_by` tokens (0 for a plain decode)
    const int short_by = h < p.H ? p.q_len - 1 - h / p.h_per_q : 0;
    const int row_len = g.len - short_by;
    // one block per iteration (a single inlined copy of softmax_block); the
    // blocks of a pass share one S buffer, released after its last read
    for (int j = g.blk_lo; j < g.blk_hi; ++j) {
      const int k = (j - g.blk_lo) % kPassBlocks;
      const bool last_of_pass = k == kPassBlocks - 1 || j + 1 == g.blk_hi;
      const int sb = pit % kNS;
      int blk;
      const int nv = block_rows(p, g, cur, j, c.lane, &blk);
      if (k == 0) {
        if (!warp_wait(bar_addr(c.bars->s_full[sb]), (pit / kNS) & 1u, c.wc)) {
          alive = false;
          break;
        }
        tc_fence_after();
      }
      const uint32_t sa = c.tmem + lane_off + kSCol + sb * kPassTok + 64 * k;
      uint32_t sv[64];
      tmem_ld32(sa, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(sa + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_ld_wait();
      if (last_of_pass) {
        tc_fence_before();
        mbar_arrive(bar_addr(c.bars->s_empty[sb]));
        ++pit;
      }
      const int nv_row = p.q_len > 1 ? max(0, min(nv, row_len - j * kBlock)) : nv;
      if (!softmax_block(c, sv, nv_row, j == g.blk_lo, sl2, pos, st, it, h, q4)) {
        alive = false;
        break;
      }
      ++it;
    }
    ++seg;
  }
  (void)alive;
}

// Sender warps (2 and 3 of the score CTA): copy each staged record into the
// value CTA with st.async (register -> remote shared memory, bytes counted on
// its p_full[r]) so that the slow SM-to-SM transfer overlaps the softmax of
// the next block.
constexpr uint32_t kRecUnits = (kPBytes + kMetaBytes) / 16;  // 16-byte units per record

__device__ void score_sender(const Ctx& c) {
  const DecodeParams& p = *c.p;
  const int sid = (c.warp - 2) * 32 + c.lane;  // 0..63
  const uint32_t prec0 = map_to_rank(c.base + p_rec_off(0), 1);
  const uint32_t mrec0 = map_to_rank(c.base + meta_rec_off(0), 1);
  const uint32_t pfull0 = map_to_rank(bar_addr(c.bars->p_full[0]), 1);
  uint32_t my_units = 0;
  for (uint32_t u = sid; u < kRecUnits; u += 64) ++my_units;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0;
  bool alive = true;
  while (alive && w.next(g)) {
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      const int r = it % kNP;
      if (!warp_wait(bar_addr(c.bars->stage_full[r]), (it / kNP) & 1u, c.wc) ||
          !warp_wait(bar_addr(c.bars->p_empty[r]), ((it / kNP) & 1u) ^ 1u, c.wc)) {
        alive = false;
        break;
      }
      const uint32_t fullr = pfull0 + 8 * r;
      mbar_arrive_expect_tx_cluster_relaxed(fullr, my_units * 16);
      const uint8_t* pst = c.gbase + p_stage_off(r);
      const uint8_t* mst = c.gbase + meta_stage_off(r);
      for (uint32_t u = sid; u < kRecUnits; u += 64) {
        if (u < kPBytes / 16) {
          const uint4 v = *reinterpret_cast<const uint4*>(pst + u * 16);
          st_async_v4(prec0 + r * kPBytes + u * 16, v, fullr);
        } else {
          const uint32_t m = u - kPBytes / 16;
          const uint4 v = *reinterpret_cast<const uint4*>(mst + m * 16);
          st_async_v4(mrec0 + r * kMetaBytes + m * 16, v, fullr);
        }
      }
      mbar_arrive(bar_addr(c.bars->stage_empty[r]));
    }
  }
  // drain: every record handed to the value CTA has been released, so no
  // remote arrival on this CTA is still pending when it exits
  if (alive) {
    for (uint32_t k = (it > kNP ? it - kNP : 0); k < it; ++k)
      if (!warp_wait(bar_addr(c.bars->p_empty[k % kNP]), (k / kNP) & 1u, c.wc)) break;
  }
}

// ============================================================ value CTA roles

__device__ void value_tma(const Ctx& c, const CUtensorMap* tmap) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  BlockCursor cur;
  uint32_t vit = 0;
  bool alive = true;
  if (c.lane == 0) prefetch_tmap(tmap);
  while (alive && w.next(g)) {
    cur.reset(p, g);
    for (int j = g.blk_lo; alive && j < g.blk_hi; ++j) {
      int blk;
      block_rows(p, g, cur, j, c.lane, &blk);
      for (int n = 0; n < 2; ++n, ++vit) {
        const int s = vit % kVSlots;
        if (!warp_wait(bar_addr(c.bars->v_empty[s]), ((vit / kVSlots) & 1u) ^ 1u, c.wc)) {
          alive = false;
          break;
        }
        if (c.lane == 0) {
          const uint32_t full = bar_addr(c.bars->v_full[s]);
          mbar_arrive_expect_tx(full, kVSlot);
          const uint32_t dst = c.base + v_slot_off(s);
#pragma unroll
          for (int q = 0; q < 4; ++q) tma_load_2d(dst + q * kChunk, tmap, (4 * n + q) * 64, blk * kBlock, full);
        }
        __syncwarp();
      }
    }
  }
  if (!alive) {
    for (uint32_t k = (vit > kVSlots ? vit - kVSlots : 0); k < vit; ++k) {
      const long long t0 = clock64();
      while (!mbar_test_wait(bar_addr(c.bars->v_full[k % kVSlots]), (k / kVSlots) & 1u) &&
             clock64() - t0 < 2000000000LL) {
      }
    }
  }
}

// Rows at or past the valid count of a block are zeroed in the V slots, so
// that whatever the cache holds there (even NaN) contributes exactly 0 * 0.
// This warp visits every slot fill (arriving on v_fixed even when nothing
// needs zeroing) so that its barrier phases stay in lockstep with the ring.
__device__ void value_fixup(const Ctx& c) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  BlockCursor cur;
  uint32_t vit = 0;
  while (w.next(g)) {
    cur.reset(p, g);
    for (int j = g.blk_lo; j < g.blk_hi; ++j) {
      int blk;
      const int nv = block_rows(p, g, cur, j, c.lane, &blk);
      for (int n = 0; n < 2; ++n, ++vit) {
        const int s = vit % kVSlots;
        if (!warp_wait(bar_addr(c.bars->v_full[s]), (vit / kVSlots) & 1u, c.wc)) return;
        if (nv < kBlock) {
          uint8_t* st = c.gbase + v_slot_off(s);
          const int rows = kBlock - nv;
          for (int idx = c.lane; idx < rows * 4 * 8; idx += 32) {
            const int ch = idx / (rows * 8);
            const int rem = idx % (rows * 8);
            const int row = nv + rem / 8;
            const int q16 = rem % 8;
            *reinterpret_cast<uint4*>(st + ch * kChunk + row * 128 + q16 * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (c.lane == 0) mbar_arrive(bar_addr(c.bars->v_fixed[s]));
      }
    }
  }
}

// As for the score MMA warp: each segment's issue loop is one single-thread
// region of lane 0.
__device__ bool value_mma_segment(const Ctx& c, const Segment& g, uint32_t seg, uint32_t& it,
                                  uint32_t& vit, uint32_t& ncorr) {
  if (seg > 0) {
    if (!wait_phase(bar_addr(c.bars->o_free), (seg - 1) & 1u, c.wc)) return false;
    tc_fence_after();
  }
  for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
    const int r = it % kNP;
    if (!wait_phase(bar_addr(c.bars->p_full[r]), (it / kNP) & 1u, c.wc)) return false;
    const bool first = (j == g.blk_lo);
    const uint8_t* meta = c.gbase + meta_rec_off(r);
    uint32_t any = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) any |= reinterpret_cast<const uint32_t*>(meta + q * kMetaWarp)[96];
    if (any && !first) {
      // hand O over for rescaling once every MMA issued so far (the previous
      // block's PV) has completed, and take it back when rescaled
      mma_commit(bar_addr(c.bars->pv_prev));
      if (!wait_phase(bar_addr(c.bars->corr_done), ncorr & 1u, c.wc)) return false;
      ++ncorr;
    }
    fence_proxy_async_smem();
    const uint32_t pa = c.base + p_rec_off(r);
    for (int n = 0; n < 2; ++n, ++vit) {
      const int s = vit % kVSlots;
      if (!wait_phase(bar_addr(c.bars->v_full[s]), (vit / kVSlots) & 1u, c.wc)) return false;
      if (!wait_phase(bar_addr(c.bars->v_fixed[s]), (vit / kVSlots) & 1u, c.wc)) return false;
      tc_fence_after();
      const uint32_t va = c.base + v_slot_off(s);
#pragma unroll
      for (int k = 0; k < kBlock / 16; ++k)
        mma_ss(c.tmem + 256 * n, sw128_desc(pa + k * 32, 16, 1024),
               sw128_desc(va + k * 2048, kChunk, 1024), kIdescPV, (k > 0 || !first) ? 1u : 0u);
      mma_commit(bar_addr(c.bars->v_empty[s]));
    }
    mma_commit_mc(bar_addr(c.bars->p_empty[r]), 0x1);
    if (j == g.blk_hi - 1) mma_commit(bar_addr(c.bars->o_ready));  // O final for this segment
  }
  return true;
}

__device__ void value_mma(const Ctx& c) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t it = 0, vit = 0, seg = 0, ncorr = 0;
  while (w.next(g)) {
    int ok = 1;
    if (c.lane == 0) ok = value_mma_segment(c, g, seg, it, vit, ncorr) ? 1 : 0;
    if (!__shfl_sync(0xffffffffu, ok, 0)) return;
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
  uint32_t it = 0, seg = 0, ncorr = 0;
  while (w.next(g)) {
    float m_fin = -INFINITY, l_fin = 0.f;
    for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
      const int r = it % kNP;
      if (!warp_wait(bar_addr(c.bars->p_full[r]), (it / kNP) & 1u, c.wc)) return;
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
      if (c.lane == 0) mbar_arrive_remote(bar_addr(c.bars->p_empty[r]), 0);
      if (any && !first) {
        // the MMA warp hands O over (pv_prev) once the previous block's PV is done
        if (!warp_wait(bar_addr(c.bars->pv_prev), ncorr & 1u, c.wc)) return;
        ++ncorr;
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
        mbar_arrive(bar_addr(c.bars->corr_done));
      }
      if (last) {
        if (!warp_wait(bar_addr(c.bars->o_ready), seg & 1u, c.wc)) return;
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
        mbar_arrive(bar_addr(c.bars->o_free));
        if (live) {
          if (g.slot < 0)
            p.lse[size_t(g.b) * p.H + h] = lse;
          else
            p.lse_part[size_t(g.slot) * p.H + h] = lse;
        }
        if (h == 0 && g.first_of_seq) p.seq_info[g.b] = seq_info_for(g, w);
      }
    }
    ++seg;
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
    for (int s = 0; s < kKSlots; ++s) {
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
      mbar_init(smem_u32(&bars->p_full[r]), 64);      // every sender thread (+ st.async bytes)
      mbar_init(smem_u32(&bars->stage_full[r]), 128); // every softmax thread
      mbar_init(smem_u32(&bars->stage_empty[r]), 64); // every sender thread
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(smem_u32(&bars->v_full[s]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 1);
      mbar_init(smem_u32(&bars->v_fixed[s]), 1);
    }
    mbar_init(smem_u32(&bars->pv_prev), 1);
    mbar_init(smem_u32(&bars->corr_done), 128);
    mbar_init(smem_u32(&bars->o_ready), 1);
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
    else if (warp <= 3) score_sender(c);
    else score_softmax(c);
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
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
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
