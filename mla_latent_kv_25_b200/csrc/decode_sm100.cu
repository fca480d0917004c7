// Absorbed MLA decode on sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// One split-KV engine = a cluster of two CTAs on two SMs, split by pipeline
// role, because the fp32 output accumulator of 128 heads x 512 latent columns
// fills all 512 TMEM columns of one SM:
//
//   score CTA (rank 0)                            value CTA (rank 1)
//   ------------------                            ------------------
//   w0    TMA: cache rows of a pass of four        w0    TMA: latent part of each block,
//         64-token blocks, two 64-column chunks          half a block (4 chunks) per slot
//         (64 KB) per ring slot                    w1    MMA: O += P V (A = P, B = V read
//   w1    MMA: S = Q K^T for 256 tokens at once          MN-major), N = 256 per instruction
//         (N = 256); Q columns 0..511 in TMEM      w2    zero V rows past seq_len
//         (TS), the RoPE columns in shared memory  w4-11 thread = (head, latent half): O
//   w4-11 softmax, thread = (head, 2 of the            rescale when a max moved; final
//         pass's 4 blocks: warps 4-7 take blocks         O / l and lse, or an fp32 piece
//         0 and 2, warps 8-11 blocks 1 and 3, so         of a cut sequence
//         that records reach the value CTA in
//         the order it consumes them): reads its
//         128 S columns at once (so the next
//         pass's QK can start), online softmax in
//         fp32, and sends P (bf16) and the
//         per-head factors straight into the value
//         CTA's shared memory (st.async)
//
// Why this shape (measured on B200): a single-CTA tcgen05.mma costs about
// 120-135 cycles to issue whatever its N up to 192, so only N = 256 runs the
// tensor pipe near its rate (the QK at ~141 cycles per 128-cycle instruction
// with A in TMEM, the PV at ~129); an mbarrier probe between MMAs stalls the
// issue stream unless it is issued ahead of the MMAs it guards, so every MMA
// loop polls the next stage's barrier before issuing the current stage; the
// SM-to-SM hand-off peaks at ~21 bytes per clock, and only when the stores
// of a warp fill whole 128-byte lines (16-byte stores to 32 different lines,
// or 32-byte sectors of them, move half as much), so P crosses without
// swizzle, in 8 x 8 core matrices: chunk c of 32 heads is 512 contiguous
// bytes.
//
// Heads are the M = 128 dimension of both contractions (padded with zero query
// rows for H < 128).  The running max of a head moves only when a pass's max
// exceeds it by more than 2^8 (log2 domain), so O is rarely rescaled; both
// softmax threads of a head take that decision on the same pass max.  Every
// wait is bounded (WaitCtx); a timeout records an error bit and the CTA leaves
// its loops, releases TMEM and exits.
//
// Barrier discipline: a parity wait can only tell the current phase from the
// one before it, so every barrier here is either observed by its waiters at
// every phase, in order, or used as a strict two-party handshake (q_ready /
// q_free, s_full / s_empty, epi_req / corr_done or o_free).
#include <cuda.h>
#include <math.h>

#include <atomic>

#include "common.cuh"
#include "kernels.h"
#include "schedule.cuh"
#include "sm100.cuh"

namespace mla {
namespace {

using namespace sm100;

constexpr int kThreads = 384;                   // warpgroup 0: TMA, MMA; warpgroups 1-2: compute
constexpr int kPassBlocks = 4;                  // score CTA: blocks per QK pass (N = 256)
constexpr int kPassTok = kPassBlocks * kBlock;
constexpr int kKSlots = 3;                      // score CTA: ring of two-chunk slots
constexpr int kFills = 5;                       // slot fills per pass: chunks {0,1} {2,3} {4,5} {6,7} {8}
constexpr int kVSlots = 4;                      // value CTA: ring of [64 x 256] half-block slots
constexpr int kNP = 5;                          // P records in flight (value CTA)

constexpr uint32_t kChunk = 64 * 128;           // [64 rows x 64 bf16] swizzled (one block, one chunk)
constexpr uint32_t kPassChunk = kPassBlocks * kChunk;  // one column chunk of a pass [256 x 64]
constexpr uint32_t kKSlot = 2 * kPassChunk;     // two column chunks of a pass
constexpr uint32_t kVSlot = 4 * kChunk;         // [64 rows x 256 bf16]
constexpr uint32_t kPBytes = 128 * 64 * 2;      // P [128 heads x 64 tokens] bf16
constexpr uint32_t kPCoreK = 128 * 16;          // P: bytes per 8-token column of core matrices
constexpr uint32_t kMetaBytes = 128 * 16;       // per head: alpha, m, l, unused
constexpr uint32_t kFlagBytes = 64;             // per quadrant: rescale flag
constexpr uint32_t kRecBytes = 19 * 1024;       // one record (P, meta, flags), 1 KB aligned
constexpr uint32_t kQTile = 128 * 64 * 2;       // [128 heads x 64] bf16 (the RoPE columns of Q)
constexpr int kQTmemChunks = 8;                 // Q columns 0..511 in TMEM (TS operand)
constexpr float kRescaleThreshold = 8.0f;       // log2 units
constexpr float kLog2e = 1.4426950408889634f;
static_assert(kPBytes + kMetaBytes + kFlagBytes <= kRecBytes, "record layout");

// TMEM columns of the score CTA: S (fp32, one column per token of the pass),
// then Q columns 0..511 as packed bf16 pairs (32 columns per 64-wide chunk).
constexpr uint32_t kSCol = 0;
constexpr uint32_t kQCol = kPassTok;
static_assert(kQCol + kQTmemChunks * 32 <= 512, "TMEM columns");
constexpr uint32_t kTmemCols = 512;

struct Barriers {
  uint64_t k_full[kKSlots], k_empty[kKSlots];
  uint64_t s_full, s_empty;
  uint64_t q_ready, q_free;
  uint64_t q_full, qstage_free;      // a segment's query tile staged by TMA
  uint64_t xchg[4];                 // softmax: the two threads of a head swap max / sum
  uint64_t p_empty[kNP];            // score CTA: record r of the value CTA is free
  uint64_t v_full[kVSlots], v_empty[kVSlots], v_fixed[kVSlots];
  uint64_t p_full[kNP];             // value CTA: record r has landed
  uint64_t epi_req, corr_done, o_free, meta_done;
  uint32_t req;                     // the MMA warp's request to the epilogue
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Barriers) <= 1024, "barrier block too large");

// shared-memory offsets from the 1024-aligned base
constexpr uint32_t kRegion = 1024;
// score CTA: exchange buffers, the RoPE tile of Q, the K ring
constexpr uint32_t kXchgOff = kRegion;                       // float [2 bufs][2 halves][128]
constexpr uint32_t kXchgBytes = 2 * 2 * 128 * 4;
constexpr uint32_t kQRopeOff = kRegion + 3072;               // 1024-aligned
__host__ __device__ constexpr uint32_t k_slot_off(int s) { return kQRopeOff + kQTile + s * kKSlot; }
constexpr uint32_t kScoreSmem = k_slot_off(kKSlots);
// each segment's query [128 rows x 512] lands by TMA in K slots 1-2 (eight
// 16 KB column chunks, 128 B swizzle) while the ring is empty, before those
// slots' next fill; its RoPE columns land straight in the RoPE tile
constexpr uint32_t kQStageOff = k_slot_off(1);
static_assert(kKSlots >= 3 && 2 * kKSlot >= 8 * kQTile, "query staging room");
// value CTA: V ring, P records
__host__ __device__ constexpr uint32_t v_slot_off(int s) { return kRegion + s * kVSlot; }
__host__ __device__ constexpr uint32_t rec_off(int r) { return kRegion + kVSlots * kVSlot + r * kRecBytes; }
constexpr uint32_t kValueSmem = rec_off(kNP);
constexpr uint32_t kSmemBytes = (kScoreSmem > kValueSmem ? kScoreSmem : kValueSmem) + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget");
static_assert(kXchgBytes <= 3072 - 0, "exchange buffers");
static_assert(kQRopeOff % 1024 == 0 && k_slot_off(0) % 1024 == 0 && rec_off(0) % 1024 == 0,
              "swizzle atoms need 1024 B");

__host__ __device__ constexpr uint32_t idesc_qk(int nb) { return idesc_bf16(128, 64 * nb, false, false); }
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

// Four consecutive blocks of a segment form one pass (fewer at the end of the
// segment); each pass streams its 9 column chunks through the slot ring, two
// chunks of all the pass's blocks per slot (the RoPE chunk alone).
__device__ void score_tma(const Ctx& c, const CUtensorMap* tmap, const CUtensorMap* qmap) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  BlockCursor cur;
  uint32_t fit = 0, seg = 0;
  bool alive = true;
  if (c.lane == 0) {
    prefetch_tmap(tmap);
    prefetch_tmap(qmap);
  }
  while (alive && w.next(g)) {
    cur.reset(p, g);
    // the segment's query tile goes to K slots 1-2 (eight latent chunks) and
    // the RoPE tile: after the previous segment's last fill has been consumed
    // (the MMAs take fills in order, so the whole ring is then free and the
    // RoPE tile no longer read)
    if (fit > 0) {
      const uint32_t k = fit - 1;
      if (!warp_wait(bar_addr(c.bars->k_empty[k % kKSlots]), (k / kKSlots) & 1u, c.wc)) {
        alive = false;
        break;
      }
    }
    if (c.lane == 0) {
      const uint32_t full = bar_addr(c.bars->q_full);
      mbar_arrive_expect_tx(full, 9 * kQTile);
      const int row = g.b * p.ld_rows;
      for (int ch = 0; ch < 8; ++ch) tma_load_2d(c.base + kQStageOff + ch * kQTile, qmap, 64 * ch, row, full);
      tma_load_2d(c.base + kQRopeOff, qmap, kDc, row, full);
    }
    __syncwarp();
    bool staged = true;  // slots 1-2 hold the query until the softmax warps took it
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
      for (int f = 0; f < kFills; ++f, ++fit) {
        const int s = fit % kKSlots;
        if (!warp_wait(bar_addr(c.bars->k_empty[s]), ((fit / kKSlots) & 1u) ^ 1u, c.wc)) {
          alive = false;
          break;
        }
        if (staged && s != 0) {
          if (!warp_wait(bar_addr(c.bars->qstage_free), seg & 1u, c.wc)) {
            alive = false;
            break;
          }
          staged = false;
        }
        if (c.lane == 0) {
          const int nch = f < 4 ? 2 : 1;
          const uint32_t full = bar_addr(c.bars->k_full[s]);
          mbar_arrive_expect_tx(full, static_cast<uint32_t>(nb * nch) * kChunk);
          const uint32_t dst = c.base + k_slot_off(s);
          for (int h = 0; h < nch; ++h)
#pragma unroll
            for (int k = 0; k < kPassBlocks; ++k)
              if (k < nb)
                tma_load_2d(dst + h * kPassChunk + k * kChunk, tmap, (2 * f + h) * 64, blk[k] * kBlock, full);
        }
        __syncwarp();
      }
    }
    ++seg;
  }
  // wait (bounded) for the loads this warp issued before the CTA may exit
  if (!alive) {
    for (uint32_t k = (fit > kKSlots ? fit - kKSlots : 0); k < fit; ++k) {
      const long long t0 = clock64();
      while (!mbar_test_wait(bar_addr(c.bars->k_full[k % kKSlots]), (k / kKSlots) & 1u) &&
             clock64() - t0 < 2000000000LL) {
      }
    }
  }
}

// The MMAs of one slot fill: chunks 2f and 2f+1 (f < 4, A from TMEM) or the
// RoPE chunk (f = 4, A from shared memory); four K = 16 steps per chunk.
__device__ __forceinline__ void qk_fill(uint32_t d, uint32_t tmem, uint32_t slot, uint32_t qrope, int f,
                                        uint32_t idesc) {
  if (f < 4) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ch = 2 * f + h;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ts(d, tmem + kQCol + 32 * ch + 8 * kk, sw128_desc(slot + h * kPassChunk + kk * 32, 16, 1024), idesc,
               (ch | kk) ? 1u : 0u);
    }
  } else {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_ss(d, sw128_desc(qrope + kk * 32, 16, 1024), sw128_desc(slot + kk * 32, 16, 1024), idesc, 1u);
  }
}

// Each segment's issue loop runs in one single-thread region of lane 0.  The
// barrier of the next slot is probed before the current slot's MMAs are
// issued, so that the probe's latency overlaps them.
__device__ bool score_mma_segment(const Ctx& c, const Segment& g, uint32_t seg, uint32_t& fit,
                                  uint32_t& pit) {
  const uint32_t tmem = c.tmem;
  const uint32_t qrope = c.base + kQRopeOff;
  const uint32_t kbase = c.base + k_slot_off(0);
  Barriers* bars = c.bars;
  if (!wait_phase(bar_addr(bars->q_ready), seg & 1u, c.wc)) return false;
  tc_fence_after();
  const int npass = (g.blk_hi - g.blk_lo + kPassBlocks - 1) / kPassBlocks;
  const int total = npass * kFills;
  // probe of fill i of this segment
  auto probe = [&](int i) -> bool {
    const uint32_t k = fit + static_cast<uint32_t>(i);
    return mbar_test_wait(bar_addr(bars->k_full[k % kKSlots]), (k / kKSlots) & 1u);
  };
  bool ready = probe(0);
  for (int ps = 0; ps < npass; ++ps, ++pit) {
    const int nb = min(kPassBlocks, g.blk_hi - g.blk_lo - ps * kPassBlocks);
    const uint32_t idesc = idesc_qk(nb);
    // S is single-buffered: the previous pass's softmax must have read it
    if (!wait_phase(bar_addr(bars->s_empty), (pit & 1u) ^ 1u, c.wc)) return false;
    tc_fence_after();
    for (int f = 0; f < kFills; ++f) {
      const uint32_t k = fit + static_cast<uint32_t>(ps * kFills + f);
      const int s = k % kKSlots;
      if (!ready && !wait_phase(bar_addr(bars->k_full[s]), (k / kKSlots) & 1u, c.wc)) return false;
      const int nxt = ps * kFills + f + 1;
      ready = nxt < total ? probe(nxt) : true;
      qk_fill(tmem + kSCol, tmem, kbase + s * kKSlot, qrope, f, idesc);
      mma_commit(bar_addr(bars->k_empty[s]));
    }
    mma_commit(bar_addr(bars->s_full));
  }
  fit += static_cast<uint32_t>(total);
  mma_commit(bar_addr(bars->q_free));
  return true;
}

__device__ void score_mma(const Ctx& c) {
  const DecodeParams& p = *c.p;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t fit = 0, pit = 0, seg = 0;
  while (w.next(g)) {
    int ok = 1;
    if (c.lane == 0) ok = score_mma_segment(c, g, seg, fit, pit) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    fit = __shfl_sync(0xffffffffu, fit, 0);
    pit = __shfl_sync(0xffffffffu, pit, 0);
    if (!ok) return;
    ++seg;
  }
}

// A segment's query row h from the TMA-staged tile: half 0 moves
// chunks 0-3 into TMEM lane h, half 1 chunks 4-7; rows at or past H (padding
// heads) get zeros, also in the RoPE tile the TMA filled.
__device__ __forceinline__ void q_half_from_stage(const Ctx& c, int h, int half, int H, uint32_t taddr,
                                                  uint8_t* qrope) {
  const bool live = h < H;
  const uint32_t swz = static_cast<uint32_t>(h & 7);
  const uint8_t* stage = c.gbase + kQStageOff + h * 128;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int ch = 4 * half + k;
    uint32_t r[32];
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const uint4 u = live ? *reinterpret_cast<const uint4*>(stage + ch * kQTile + ((static_cast<uint32_t>(v) ^ swz) << 4))
                           : make_uint4(0, 0, 0, 0);
      r[4 * v] = u.x;
      r[4 * v + 1] = u.y;
      r[4 * v + 2] = u.z;
      r[4 * v + 3] = u.w;
    }
    tmem_st32(taddr + kQCol + 32 * ch, r);
  }
  if (half == 1 && !live) {
#pragma unroll
    for (int v = 0; v < 8; ++v) *reinterpret_cast<uint4*>(qrope + h * 128 + v * 16) = make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void prefetch_q_row_l2(const DecodeParams& p, int b, int h) {
  if (h >= p.H) return;
  const char* src = reinterpret_cast<const char*>(p.q + (size_t(b) * p.ld_rows + h) * kRow);
#pragma unroll
  for (int i = 0; i < 9; ++i) asm volatile("prefetch.global.L2 [%0];" ::"l"(src + 128 * i));
}

// Swap a float with the other softmax thread of the same head (same quadrant,
// other half) through shared memory and the quadrant's exchange barrier.
__device__ __forceinline__ bool xchg(const Ctx& c, int q4, int half, int h, uint32_t& xit, float mine,
                                     float* other) {
  float* buf = reinterpret_cast<float*>(c.gbase + kXchgOff) + (xit & 1u) * 256;
  buf[half * 128 + h] = mine;
  mbar_arrive(bar_addr(c.bars->xchg[q4]));
  if (!warp_wait(bar_addr(c.bars->xchg[q4]), xit & 1u, c.wc)) return false;
  *other = buf[(half ^ 1) * 128 + h];
  ++xit;
  return true;
}

__device__ void score_softmax(const Ctx& c) {
  const DecodeParams& p = *c.p;
  const int q4 = c.warp & 3;              // TMEM lane quadrant (a warp reaches lanes 32*(warp%4)..)
  const int half = (c.warp - 4) >> 2;     // blocks half, half + 2 of each pass
  const int h = q4 * 32 + c.lane;         // head of this thread
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  // a zero scale (uniform attention) runs as a tiny one, so that a masked
  // score (-inf) still gives exactly 0 (scores then differ by < 1e-27)
  const float sl2 = p.softmax_scale != 0.f ? p.softmax_scale * kLog2e : 1e-30f;
  const bool pos = sl2 >= 0.f;
  const float sg = pos ? 1.f : -1.f;
  uint8_t* qrope = c.gbase + kQRopeOff;
  const uint32_t rec0 = map_to_rank(c.base + rec_off(0), 1);
  const uint32_t pfull0 = map_to_rank(bar_addr(c.bars->p_full[0]), 1);
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  BlockCursor cur;
  uint32_t it = 0, pit = 0, seg = 0, xit = 0;
  bool alive = true;
  while (alive && w.next(g)) {
    cur.reset(p, g);
    if (seg > 0) {
      if (!warp_wait(bar_addr(c.bars->q_free), (seg - 1) & 1u, c.wc)) break;
      tc_fence_after();
    }
    if (!warp_wait(bar_addr(c.bars->q_full), seg & 1u, c.wc)) break;
    q_half_from_stage(c, h, half, p.H, c.tmem + lane_off, qrope);
    __syncwarp();
    if (c.lane == 0) mbar_arrive(bar_addr(c.bars->qstage_free));
    fence_proxy_async_smem();
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(bar_addr(c.bars->q_ready));
    if (w.b < w.B && w.pre < w.e) prefetch_q_row_l2(p, w.b, h);  // next segment's query

    float m_ref = -INFINITY, l = 0.f;
    // multi-token decode: this row's query token sees the sequence without
    // its last `short_by` tokens (0 for a plain decode)
    const int short_by = h < p.H ? p.q_len - 1 - h / p.h_per_q : 0;
    const int row_len = g.len - short_by;
    for (int j0 = g.blk_lo; j0 < g.blk_hi; j0 += kPassBlocks, ++pit) {
      const bool first_pass = (j0 == g.blk_lo);
      const int nb = min(kPassBlocks, g.blk_hi - j0);
      // the two blocks of this thread in the pass (absent ones have no rows)
      int nvr[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int kb = half + 2 * k;
        int blk;
        // every lane of the warp takes part in the cursor's shuffle
        const int nv = block_rows(p, g, cur, kb < nb ? j0 + kb : j0, c.lane, &blk);
        const int jj = j0 + kb;
        int nr = kb < nb ? nv : 0;
        if (p.q_len > 1) nr = max(0, min(nr, row_len - jj * kBlock));
        nvr[k] = nr;
      }
      if (!warp_wait(bar_addr(c.bars->s_full), pit & 1u, c.wc)) {
        alive = false;
        break;
      }
      tc_fence_after();
      uint32_t sv[128];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        tmem_ld32(c.tmem + lane_off + kSCol + 64 * half + 128 * (q >> 1) + 32 * (q & 1),
                  *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * q]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(bar_addr(c.bars->s_empty));

      // columns at or past a block's valid count (rare: the last block of a
      // sequence, absent blocks of a short pass) take the score -sg * inf,
      // which no max selects; the exponentials below mask them explicitly
      if (!__all_sync(0xffffffffu, nvr[0] == kBlock && nvr[1] == kBlock)) {
        const uint32_t masked = __float_as_uint(-INFINITY * sg);
#pragma unroll
        for (int t = 0; t < 128; ++t)
          if ((t & 63) >= nvr[t >> 6]) sv[t] = masked;
      }
      // pass max of the scaled scores over both threads of the head: max of
      // s * sg with sg = sign(scale), so a negative scale needs no second
      // code path
      float mr;
      if (pos) {
        float mv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int t = 0; t < 128; t += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            mv[u] = fmax3(mv[u], __uint_as_float(sv[t + 2 * u]), __uint_as_float(sv[t + 2 * u + 1]));
        mr = fmax3(fmaxf(mv[0], mv[1]), mv[2], mv[3]);
      } else {
        float mv[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll
        for (int t = 0; t < 128; t += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            mv[u] = fmin3(mv[u], __uint_as_float(sv[t + 2 * u]), __uint_as_float(sv[t + 2 * u + 1]));
        mr = -fmin3(fminf(mv[0], mv[1]), mv[2], mv[3]);
      }
      const float mine = (nvr[0] | nvr[1]) ? mr * sg * sl2 : -INFINITY;
      float other;
      if (!xchg(c, q4, half, h, xit, mine, &other)) {
        alive = false;
        break;
      }
      const float mx = fmaxf(mine, other);
      float alpha = 1.f;
      bool resc = false;
      if (first_pass) {
        m_ref = mx;
      } else if (mx > m_ref + kRescaleThreshold) {
        alpha = (m_ref == -INFINITY) ? 0.f : ex2_approx(m_ref - mx);
        m_ref = mx;
        l *= alpha;
        resc = true;
      }
      const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
      const unsigned any = __any_sync(0xffffffffu, resc);

      // P rows of this thread's blocks straight into the value CTA's records.
      // Columns past a block's valid count hold -sg * inf, whose exponential
      // is exactly 0 (sl2 is never 0), so no masking is needed here.
      const bool last_pass = j0 + kPassBlocks >= g.blk_hi;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int kb = half + 2 * k;
        if (kb >= nb) continue;
        const uint32_t ib = it + static_cast<uint32_t>(kb);
        const int r = ib % kNP;
        if (!warp_wait(bar_addr(c.bars->p_empty[r]), ((ib / kNP) & 1u) ^ 1u, c.wc)) {
          alive = false;
          break;
        }
        const uint32_t full = pfull0 + 8 * r;
        const uint32_t rec = rec0 + r * kRecBytes;
        // one remote arrival per warp announces the warp's bytes: each lane's
        // P row (128) and, for a pass's first block and the segment's last,
        // its factors (16); lane 0's rescale flag (4)
        const bool meta = kb == 0 || (last_pass && kb == nb - 1);
        if (c.lane == 0) mbar_arrive_expect_tx_cluster_relaxed(full, 32 * (128 + (meta ? 16 : 0)) + 4);
        float sum0 = 0.f, sum1 = 0.f;
        // the record holds P without swizzle in 8 x 8 core matrices (token
        // chunk c of heads 8i..8i+7 in 128 contiguous bytes): the 32 lanes'
        // 16-byte chunks c of one warp fill four whole 128-byte lines
#pragma unroll
        for (int tp = 0; tp < 4; ++tp) {
          uint32_t pk[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int t = 64 * k + 16 * tp + 8 * u + 2 * e;
              const float e0 = ex2_approx(fmaf(__uint_as_float(sv[t]), sl2, neg_m));
              const float e1 = ex2_approx(fmaf(__uint_as_float(sv[t + 1]), sl2, neg_m));
              sum0 += e0;
              sum1 += e1;
              __nv_bfloat162 b2 = __floats2bfloat162_rn(e0, e1);
              pk[u][e] = *reinterpret_cast<uint32_t*>(&b2);
            }
#pragma unroll
          for (int u = 0; u < 2; ++u)
            st_async_v4(rec + (2 * tp + u) * kPCoreK + h * 16, make_uint4(pk[u][0], pk[u][1], pk[u][2], pk[u][3]),
                        full);
        }
        l += sum0 + sum1;
        if (c.lane == 0) st_async_b32(rec + kPBytes + kMetaBytes + q4 * 4, (kb == 0 && any) ? 1u : 0u, full);
        // a pass's first block carries the pass's rescale factor; unless it
        // is also the segment's last block, its factors are final now
        if (kb == 0 && !(last_pass && nb == 1))
          st_async_v4(rec + kPBytes + h * 16,
                      make_uint4(__float_as_uint(alpha), __float_as_uint(m_ref), __float_as_uint(l), 0u), full);
      }
      if (!alive) break;
      // factors: the rescale factor of the pass (its first block's record)
      // and, with the segment's last block, the running max and the sum over
      // both threads of the head
      float ltot = l;
      if (last_pass) {
        float lo;
        if (!xchg(c, q4, half, h, xit, l, &lo)) {
          alive = false;
          break;
        }
        ltot = l + lo;
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int kb = half + 2 * k;
        if (!(last_pass && kb == nb - 1)) continue;
        const uint32_t ib = it + static_cast<uint32_t>(kb);
        const int r = ib % kNP;
        st_async_v4(rec0 + r * kRecBytes + kPBytes + h * 16,
                    make_uint4(__float_as_uint(kb == 0 ? alpha : 1.f), __float_as_uint(m_ref),
                               __float_as_uint(ltot), 0u),
                    pfull0 + 8 * r);
      }
      if (!alive) break;
      it += static_cast<uint32_t>(nb);
    }
    ++seg;
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

// As for the score MMA warp: each segment's issue loop runs in one
// single-thread region of lane 0, and the next slot's barrier is probed
// before the current slot's MMAs are issued.  The epilogue warps act only on
// requests: a rescale of O before a record's PV, and the final output after
// the segment's last PV (kReqFinal | record), each posted in `req` with a
// plain arrival on epi_req plus a commit (the MMAs issued so far are done).
constexpr uint32_t kReqFinal = 0x80000000u;

__device__ __forceinline__ void post_request(const Ctx& c, uint32_t req) {
  *reinterpret_cast<volatile uint32_t*>(&c.bars->req) = req;
  mbar_arrive(bar_addr(c.bars->epi_req));
  mma_commit(bar_addr(c.bars->epi_req));
}

__device__ bool value_mma_segment(const Ctx& c, const Segment& g, uint32_t seg, uint32_t& it,
                                  uint32_t& vit, uint32_t& ncorr) {
  if (seg > 0) {
    if (!wait_phase(bar_addr(c.bars->o_free), (seg - 1) & 1u, c.wc)) return false;
    tc_fence_after();
  }
  bool ready = mbar_test_wait(bar_addr(c.bars->v_fixed[vit % kVSlots]), (vit / kVSlots) & 1u);
  for (int j = g.blk_lo; j < g.blk_hi; ++j, ++it) {
    const int r = it % kNP;
    if (!wait_phase(bar_addr(c.bars->p_full[r]), (it / kNP) & 1u, c.wc)) return false;
    const bool first = (j == g.blk_lo);
    const bool last = (j == g.blk_hi - 1);
    const uint32_t* flags = reinterpret_cast<const uint32_t*>(c.gbase + rec_off(r) + kPBytes + kMetaBytes);
    const uint32_t any = flags[0] | flags[1] | flags[2] | flags[3];
    if (any && !first) {
      // hand O over for rescaling once every MMA issued so far (the previous
      // blocks' PV) has completed, and take it back when rescaled
      post_request(c, static_cast<uint32_t>(r));
      if (!wait_phase(bar_addr(c.bars->corr_done), ncorr & 1u, c.wc)) return false;
      ++ncorr;
      tc_fence_after();
    }
    fence_proxy_async_smem();
    const uint32_t pa = c.base + rec_off(r);
    for (int n = 0; n < 2; ++n, ++vit) {
      const int s = vit % kVSlots;
      // v_fixed completes after v_full (the fixup warp waits v_full first)
      if (!ready && !wait_phase(bar_addr(c.bars->v_fixed[s]), (vit / kVSlots) & 1u, c.wc)) return false;
      const uint32_t nx = vit + 1;
      ready = mbar_test_wait(bar_addr(c.bars->v_fixed[nx % kVSlots]), (nx / kVSlots) & 1u);
      const uint32_t va = c.base + v_slot_off(s);
#pragma unroll
      for (int k = 0; k < kBlock / 16; ++k)
        mma_ss(c.tmem + 256 * n, plain_desc(pa + k * 2 * kPCoreK, kPCoreK, 128),
               sw128_desc(va + k * 2048, kChunk, 1024), kIdescPV, (k > 0 || !first) ? 1u : 0u);
      mma_commit(bar_addr(c.bars->v_empty[s]));
    }
    if (last)
      post_request(c, kReqFinal | static_cast<uint32_t>(r));  // the epilogue releases the record
    else
      mma_commit_mc(bar_addr(c.bars->p_empty[r]), 0x1);
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

// Thread = (head h, latent half): the rescales and the final normalisation
// of O's 256 columns [256 * half, 256 * half + 256) of TMEM lane h, on the
// MMA warp's requests.
__device__ void value_epilogue(const Ctx& c) {
  const DecodeParams& p = *c.p;
  const int q4 = c.warp & 3;
  const int half = (c.warp - 4) >> 2;
  const int h = q4 * 32 + c.lane;
  const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
  const uint32_t ocol = 256 * half;
  SegWalker w;
  w.init(p.seq_lens, p.B, p.max_blocks, p.P, c.engine);
  Segment g;
  uint32_t nreq = 0, nfinal = 0;
  while (w.next(g)) {
    for (;;) {
      if (!warp_wait(bar_addr(c.bars->epi_req), nreq & 1u, c.wc)) return;
      ++nreq;
      tc_fence_after();
      const uint32_t req = *reinterpret_cast<volatile uint32_t*>(&c.bars->req);
      const uint8_t* rec = c.gbase + rec_off(static_cast<int>(req & 0xffu));
      const float4 meta = *reinterpret_cast<const float4*>(rec + kPBytes + h * 16);
      if (!(req & kReqFinal)) {
        const float alpha = meta.x;
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t v[32];
          tmem_ld32(c.tmem + lane_off + ocol + 32 * ch, v);
          tmem_ld_wait();
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = __float_as_uint(__uint_as_float(v[t]) * alpha);
          tmem_st32(c.tmem + lane_off + ocol + 32 * ch, v);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_addr(c.bars->corr_done));
        continue;
      }
      // final: O / l and lse (or the fp32 piece of a cut sequence).  The
      // record goes back to the score CTA once all eight warps have read it.
      const float m_fin = meta.y, l_fin = meta.z;
      __syncwarp();
      if (c.lane == 0) mbar_arrive(bar_addr(c.bars->meta_done));
      if (c.warp == 4) {
        if (!warp_wait(bar_addr(c.bars->meta_done), nfinal & 1u, c.wc)) return;
        if (c.lane == 0) mbar_arrive_remote(bar_addr(c.bars->p_empty[req & 0xffu]), 0);
      }
      ++nfinal;
      const bool live = h < p.H;
      const float inv = l_fin > 0.f ? 1.f / l_fin : 0.f;
      const float lse = l_fin > 0.f ? (m_fin + log2f(l_fin)) * 0.6931471805599453f : -INFINITY;
#pragma unroll 1
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t v[32];
        tmem_ld32(c.tmem + lane_off + ocol + 32 * ch, v);
        tmem_ld_wait();
        if (!live) continue;
        const int col = ocol + 32 * ch;
        if (g.slot < 0) {
          uint4* dst = reinterpret_cast<uint4*>(p.out + (size_t(g.b) * p.ld_rows + h) * kDc + col);
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
          float4* dst = reinterpret_cast<float4*>(p.o_part + (size_t(g.slot) * p.H + h) * kDc + col);
#pragma unroll
          for (int q = 0; q < 8; ++q)
            dst[q] = make_float4(__uint_as_float(v[4 * q]) * inv, __uint_as_float(v[4 * q + 1]) * inv,
                                 __uint_as_float(v[4 * q + 2]) * inv, __uint_as_float(v[4 * q + 3]) * inv);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_addr(c.bars->o_free));
      if (live && half == 0) {
        if (g.slot < 0)
          p.lse[size_t(g.b) * p.ld_rows + h] = lse;
        else
          p.lse_part[size_t(g.slot) * p.H + h] = lse;
      }
      if (h == 0 && half == 0 && g.first_of_seq) p.seq_info[g.b] = seq_info_for(g, w);
      break;
    }
  }
}

// ============================================================ kernel

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
decode_sm100_kernel(const __grid_constant__ CUtensorMap tmap, const __grid_constant__ CUtensorMap qmap,
                    const DecodeParams p) {
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
    mbar_init(smem_u32(&bars->s_full), 1);
    mbar_init(smem_u32(&bars->s_empty), 256);       // every softmax thread
    mbar_init(smem_u32(&bars->q_ready), 256);
    mbar_init(smem_u32(&bars->q_free), 1);
    mbar_init(smem_u32(&bars->q_full), 1);
    mbar_init(smem_u32(&bars->qstage_free), 8);     // lane 0 of every softmax warp
    for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&bars->xchg[q]), 64);  // two warps
    for (int r = 0; r < kNP; ++r) {
      mbar_init(smem_u32(&bars->p_empty[r]), 1);      // PV commit, or the epilogue (segment end)
      mbar_init(smem_u32(&bars->p_full[r]), 4);       // the four softmax warps of one half
    }
    for (int s = 0; s < kVSlots; ++s) {
      mbar_init(smem_u32(&bars->v_full[s]), 1);
      mbar_init(smem_u32(&bars->v_empty[s]), 1);
      mbar_init(smem_u32(&bars->v_fixed[s]), 1);
    }
    mbar_init(smem_u32(&bars->epi_req), 2);         // request word posted + commit
    mbar_init(smem_u32(&bars->corr_done), 256);
    mbar_init(smem_u32(&bars->o_free), 256);
    mbar_init(smem_u32(&bars->meta_done), 8);        // every epilogue warp read the final record
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
  // launched with programmatic stream serialization: the set-up above ran
  // while the previous kernel on the stream finished; every global read and
  // write comes after this wait.  The merge kernel that follows may be
  // scheduled now (it waits for this grid to complete before its work).
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  Ctx c;
  c.p = &p;
  c.base = base;
  c.gbase = gbase;
  c.bars = bars;
  c.tmem = bars->tmem_base;
  c.wc = WaitCtx{p.spin_limit, p.err, &bars->abort, p.err + 1};
  c.engine = blockIdx.x >> 1;
  c.warp = warp;
  c.lane = lane;

  if (warp < 4) {
    if (rank == 0) {
      if (warp == 0) score_tma(c, &tmap, &qmap);
      else if (warp == 1) score_mma(c);
    } else {
      if (warp == 0) value_tma(c, &tmap);
      else if (warp == 1) value_mma(c);
      else if (warp == 2) value_fixup(c);
    }
  } else {
    if (rank == 0) score_softmax(c);
    else value_epilogue(c);
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

cudaError_t launch_decode_sm100(const DecodeParams& p, const CUtensorMap& tmap, const CUtensorMap& qmap,
                                cudaStream_t stream) {
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(decode_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_set[dev].store(true, std::memory_order_release);
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * p.P);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_sm100_kernel, tmap, qmap, p);
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
