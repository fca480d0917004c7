// Host-side check of the split-KV partition and workspace layout the decode
// kernels use (common.cuh), compiled and run by tests/test_partition.py.
// Prints "ok <cases>" or the first violated property.
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "../mla_latent_kv_25_b200/csrc/common.cuh"
#include "../mla_latent_kv_25_b200/csrc/plan.h"

using namespace mla;

static unsigned long long rng = 88172645463325252ull;
static unsigned long long next() { rng ^= rng << 13; rng ^= rng >> 7; rng ^= rng << 17; return rng; }

#define CHECK(c, ...) do { if (!(c)) { std::printf(__VA_ARGS__); std::printf("\n"); return 1; } } while (0)

int main() {
  int cases = 0;
  for (int it = 0; it < 3000; ++it) {
    const long long NBt = 1 + static_cast<long long>(next() % (it < 1000 ? 300 : 2000000));
    const int Pmax = static_cast<int>(NBt < 4096 ? NBt : 4096);
    const int P = 1 + static_cast<int>(next() % Pmax);   // the library never uses more engines than blocks
    // ranges: contiguous, non-empty, covering [0, NBt)
    CHECK(range_start(0, NBt, P) == 0, "start(0) != 0");
    CHECK(range_start(P, NBt, P) == NBt, "start(P) != NBt (NBt=%lld P=%d)", NBt, P);
    for (int p = 0; p < P; ++p)
      CHECK(range_start(p + 1, NBt, P) > range_start(p, NBt, P), "empty range p=%d NBt=%lld P=%d", p, NBt, P);
    // engine_of inverts the ranges at every range boundary and at sampled blocks
    for (int p = 0; p < P; ++p) {
      const long long s = range_start(p, NBt, P), e = range_start(p + 1, NBt, P);
      CHECK(engine_of(s, NBt, P) == p, "engine_of(start) p=%d", p);
      CHECK(engine_of(e - 1, NBt, P) == p, "engine_of(end-1) p=%d", p);
      const long long x = s + static_cast<long long>(next() % static_cast<unsigned long long>(e - s));
      CHECK(engine_of(x, NBt, P) == p, "engine_of(x) p=%d", p);
    }
    ++cases;
  }
  // sequences laid end to end: each sequence's pieces sit on consecutive
  // engines p0..p1, and an engine holds at most two cut pieces (its first and
  // last segment), the property the merge relies on
  for (int it = 0; it < 500; ++it) {
    const int B = 1 + static_cast<int>(next() % 300);
    std::vector<long long> nb(B);
    long long NBt = 0;
    for (int b = 0; b < B; ++b) { nb[b] = static_cast<long long>(next() % 200); NBt += nb[b]; }
    if (NBt == 0) continue;
    const int P = 1 + static_cast<int>(next() % (NBt < 600 ? NBt : 600));
    std::vector<int> cut_pieces(P, 0);
    long long pre = 0;
    for (int b = 0; b < B; ++b) {
      if (nb[b] == 0) continue;
      const int p0 = engine_of(pre, NBt, P), p1 = engine_of(pre + nb[b] - 1, NBt, P);
      CHECK(p0 <= p1, "engines out of order");
      if (p1 > p0) {
        for (int p = p0; p <= p1; ++p) ++cut_pieces[p];
        // every engine after the first starts its range inside this sequence:
        // the piece is its first segment
        for (int p = p0 + 1; p <= p1; ++p)
          CHECK(range_start(p, NBt, P) > pre && range_start(p, NBt, P) < pre + nb[b], "piece not first segment");
      }
      pre += nb[b];
    }
    for (int p = 0; p < P; ++p) CHECK(cut_pieces[p] <= 2, "engine %d holds %d cut pieces", p, cut_pieces[p]);
    ++cases;
  }
  // workspace layout: 256-byte aligned, disjoint, large enough
  for (int it = 0; it < 1000; ++it) {
    const int B = 1 + static_cast<int>(next() % 100000), H = 16 * (1 + static_cast<int>(next() % 8));
    const int P = 1 + static_cast<int>(next() % 4096);
    const WsLayout w = ws_layout(B, H, P);
    CHECK(w.seq_info % 256 == 0 && w.lse_part % 256 == 0 && w.o_part % 256 == 0 && w.total % 256 == 0, "alignment");
    CHECK(w.seq_info >= 4 && w.lse_part >= w.seq_info + size_t(B) * 16, "seq_info overlaps");
    CHECK(w.o_part >= w.lse_part + size_t(2 * P) * H * 4, "lse_part overlaps");
    CHECK(w.total >= w.o_part + size_t(2 * P) * H * kDc * 4, "o_part overflows");
    ++cases;
  }
  // fp8 decode groups (plan.h): every group fits the workspace, the groups
  // cover the batch, the whole batch at the requested engine count when it
  // fits, and no plan only when not even one sequence on one engine fits
  for (int it = 0; it < 4000; ++it) {
    const int B = 1 + static_cast<int>(next() % 300);
    const int rows = 16 * (1 + static_cast<int>(next() % 8));
    const int mb = 1 + static_cast<int>(next() % (it % 4 == 0 ? 4096 : 256));
    const int cap = 1 + static_cast<int>(next() % 148);
    auto engines_for = [&](int n) { return n < cap ? n : cap; };
    const int P = engines_for(B);
    const size_t whole = fp8_group_bytes(B, rows, mb, P);
    const size_t one = fp8_group_bytes(1, rows, mb, 1);
    size_t ws = 0;
    switch (it % 4) {
      case 0: ws = whole; break;                                    // exactly the whole batch
      case 1: ws = one + next() % (whole > one ? whole - one : 1); break;  // between
      case 2: ws = one > 0 ? one - 1 - next() % (one < 1000 ? one : 1000) : 0; break;  // too small
      default: ws = static_cast<size_t>(next() % (whole + 1)); break;
    }
    const Fp8Plan plan = plan_fp8_groups(B, rows, mb, P, ws, engines_for);
    if (plan.Bg == 0) {
      CHECK(one == 0 || one > ws, "no plan although one sequence fits (B=%d mb=%d ws=%zu one=%zu)", B, mb, ws, one);
      continue;
    }
    CHECK(plan.Bg >= 1 && plan.Bg <= B && plan.Pg >= 1, "plan out of range Bg=%d Pg=%d", plan.Bg, plan.Pg);
    if (whole != 0 && whole <= ws) CHECK(plan.Bg == B && plan.Pg == P, "whole batch fits but Bg=%d Pg=%d", plan.Bg, plan.Pg);
    int covered = 0;
    for (int b0 = 0; b0 < B; b0 += plan.Bg) {
      const int n = B - b0 < plan.Bg ? B - b0 : plan.Bg;
      const int pg = plan.Pg < engines_for(n) ? plan.Pg : engines_for(n);
      const size_t need = fp8_group_bytes(n, rows, mb, pg);
      CHECK(need != 0 && need <= ws, "group at %d (n=%d, %d engines) needs %zu > %zu", b0, n, pg, need, ws);
      covered += n;
    }
    CHECK(covered == B, "groups cover %d of %d", covered, B);
    ++cases;
  }
  std::printf("ok %d\n", cases);
  return 0;
}
