// Host-side checks of the tcgen05 kernel's tile logic (compiled with nvcc for
// sm_100a, runs on the CPU only; no CUDA call is made):
//   * the tile walk: every kept row of every pattern is in exactly one tile,
//     tiles come in the combination order (start position, larger r first,
//     pattern index), every position is finalised exactly once (by the last
//     tile covering it), and no pattern's parking slot is overwritten while
//     it still holds a row;
//   * TMA coordinates of every Q tile and K/V block address exactly the kept
//     rows they should, inside the tensor;
//   * the multiply-shift divider equals integer division, and the coverage
//     test that uses it equals the plain one.
#include "tcgen05.cu"

#include <cstdio>
#include <vector>
#include <map>
#include <set>
#include <tuple>

using namespace longnet;
using namespace longnet::tc;

static int fails = 0;
#define CHECK(c, ...)                    \
  do {                                   \
    if (!(c)) {                          \
      if (fails < 20) printf(__VA_ARGS__); \
      ++fails;                           \
    }                                    \
  } while (0)

void check_tma(const Params& P, int ri, int64_t first, int64_t need, int64_t r) {
  TmaCoord c = tma_coord(P, ri, first, need);
  for (int64_t i = 0; i < need; ++i) {
    int64_t pos;
    if (c.map == 0) {
      CHECK(c.c >= 0 && c.c < r, "map0 c out of range\n");
      CHECK(c.kk + i < P.kfull[ri] && c.kk >= 0, "map0 k oob first=%ld need=%ld i=%ld\n", (long)first, (long)need, (long)i);
      pos = r * (c.kk + i) + c.c;
    } else {
      CHECK(c.c >= 0 && c.c < r, "map1 c out of range\n");
      CHECK(c.kk + i < P.kfull[ri] && c.kk >= 0, "map1 k oob\n");
      pos = P.tail[ri] + r * (c.kk + i) + c.c;
    }
    CHECK(pos == first + r * i, "tma pos mismatch %ld vs %ld\n", (long)pos, (long)(first + r * i));
  }
}

bool run_case(const char* name, int64_t B, int64_t N, int64_t H, std::vector<std::pair<int64_t, int64_t>> pats, int causal,
              int sms = 148, bool quiet = false, int64_t q0 = 0, int64_t q1 = -1, int64_t h0 = 0, int64_t h1 = -1) {
  Problem pb;
  memset(&pb, 0, sizeof(pb));
  pb.B = B; pb.N = N; pb.H = H; pb.D = 64; pb.n_pat = (int)pats.size(); pb.causal = causal;
  pb.dtype = LONGNET_DTYPE_BF16;
  for (int i = 0; i < pb.n_pat; ++i) { pb.w[i] = pats[i].first; pb.r[i] = pats[i].second; }
  pb.q0 = q0;
  pb.q1 = q1 < 0 ? N : q1;
  pb.h0 = h0;
  pb.h1 = h1 < 0 ? H : h1;
  if (!tcgen05_supports(pb)) {
    if (!quiet) printf("%s: not supported\n", name);
    return false;
  }
  static Params P;
  fill_params(pb, P, sms);
  int f0 = fails;
  long n_tiles = 0, n_kv = 0;
  // coverage: (p, h, seg, k) -> count
  for (int64_t h = pb.h0; h < pb.h1; ++h) {
    std::map<std::tuple<int, int64_t, int64_t>, int> seen;
    std::vector<int> finalized(N, 0);
    for (int rank = 0; rank < P.n_units; ++rank) {
      int A32, B32;
      unit_bounds(P, rank, A32, B32);
      const int64_t A = A32, Bnd = B32;
      CHECK(A >= pb.q0 && Bnd <= pb.q1, "%s: unit [%ld, %ld) outside the part\n", name, (long)A, (long)Bnd);
      {
        // the TMA threads' fast block sequence equals the reference one, and
        // a stream never starts a tile whose O buffer's previous user still
        // has blocks behind the other stream's
        BlockSeq bs;
        bs.init(P, (int)h, (int)A, (int)Bnd);
        TileWalker tw2;
        tw2.init(P, h, A, Bnd);
        FastSeq fs;
        fs.init(&tw2, block_cost(ring_stages(P.stages, 0)), block_cost(ring_stages(P.stages, 1)));
        Elem e1, e2;
        long n_elem = 0, per_stream[2] = {0, 0};
        for (;;) {
          const bool a = bs.next(e1), b = fs.next(e2);
          CHECK(a == b, "%s: block sequences end differently\n", name);
          if (!a || !b) break;
          CHECK(e1.g == e2.g && e1.j == e2.j && e1.tile_idx == e2.tile_idx && e1.ob == e2.ob &&
                    e1.use == e2.use && e1.t.start == e2.t.start && e1.t.p == e2.t.p && e1.t.nkv == e2.t.nkv,
                "%s: block %ld of the fast sequence differs from the reference\n", name, n_elem);
          ++n_elem;
          ++per_stream[e1.g];
        }
        (void)per_stream;
      }
      TileWalker tw;
      tw.init(P, h, A, Bnd);
      Tile t;
      // slot state: pattern -> (tile start, set of rows still waiting)
      std::map<int, int64_t> slot_tile_start;
      std::map<int, std::set<int64_t>> slot_pending;  // positions parked
      int64_t prev_key_start = -1, prev_r = 0; int prev_p = -1;
      while (tw.next(t)) {
        ++n_tiles; n_kv += t.nkv;
        CHECK(t.nrows >= 1 && t.nrows <= 128, "bad nrows\n");
        if (prev_p >= 0) CHECK(key_before(prev_key_start, prev_r, prev_p, t.start, tw.r[t.p], t.p), "order violated\n");
        prev_key_start = t.start; prev_r = tw.r[t.p]; prev_p = t.p;
        const int64_t r = tw.r[t.p];
        const int64_t base = t.seg * tw.w[t.p] + tw.o[t.p];
        CHECK(t.start == base + r * t.k0, "start mismatch\n");
        // keys: the kept rows of the segment (before the sequence's end), up
        // to the tile's last row when causal
        const int64_t seg_end = std::min<int64_t>((t.seg + 1) * (int64_t)tw.w[t.p], N);
        int64_t seg_kept = 0;
        for (int64_t xk = base; xk < seg_end; xk += r) ++seg_kept;
        int64_t nkeys = causal ? t.k0 + t.nrows : seg_kept;
        CHECK(t.k0 + t.nrows <= seg_kept, "%s: tile rows past the segment's kept rows\n", name);
        CHECK(t.nkeys == nkeys, "%s: nkeys %d, expected %ld\n", name, t.nkeys, (long)nkeys);
        CHECK(t.nkv == (nkeys + kBN - 1) / kBN, "nkv\n");
        // TMA coords
        check_tma(P, P.pat_r[t.p], t.start, t.nrows, r);
        for (int j = 0; j < t.nkv; ++j) {
          int64_t need = std::min<int64_t>(kBN, nkeys - kBN * j);
          check_tma(P, P.pat_r[t.p], base + r * kBN * j, need, r);
        }
        // slot overwrite check: previous tile of this pattern fully consumed
        CHECK(slot_pending[t.p].empty(), "%s: slot of pattern %d overwritten with %zu rows pending\n", name, t.p, slot_pending[t.p].size());
        slot_tile_start[t.p] = t.start;
        for (int row = 0; row < t.nrows; ++row) {
          int64_t k = t.k0 + row;
          auto key = std::make_tuple(t.p, t.seg, k);
          seen[key]++;
          int64_t x = t.start + r * row;
          CHECK(x >= A && x < Bnd, "row outside range\n");
          CHECK(x == base + r * k, "pos\n");
          bool final_row = true;
          for (int q = 0; q < tw.n_pat; ++q) {
            Cover cv, cf;
            const bool c1 = cover_of(tw, q, x, cv);
            const bool c2 = cover_pat_fd(tw.w[q], tw.r[q], tw.o[q], tw.m[q], tw.A, x, P.w_div[q],
                                         P.r_div[P.pat_r[q]], cf);
            CHECK(c1 == c2 && (!c1 || (cv.start == cf.start && cv.slot_row == cf.slot_row)),
                  "%s: fast coverage differs q=%d x=%ld\n", name, q, (long)x);
            if (q == t.p) continue;
            if (!c1) continue;
            if (!key_before(cv.start, tw.r[q], q, t.start, tw.r[t.p], t.p)) final_row = false;
          }
          if (final_row) {
            for (int q = 0; q < tw.n_pat; ++q) {
              if (q == t.p) continue;
              Cover cv;
              if (!cover_of(tw, q, x, cv)) continue;
              CHECK(slot_tile_start.count(q) && slot_tile_start[q] == cv.start, "%s: finalizer reads stale slot q=%d\n", name, q);
              CHECK(slot_pending[q].count(x) == 1, "%s: parked row missing q=%d x=%ld\n", name, q, (long)x);
              CHECK(cv.start + tw.r[q] * cv.slot_row == x, "slot row mismatch\n");
              slot_pending[q].erase(x);
            }
            finalized[x]++;
          } else {
            slot_pending[t.p].insert(x);
          }
        }
      }
      for (auto& kv : slot_pending) CHECK(kv.second.empty(), "%s: rows left parked at unit end\n", name);
    }
    // every kept row exactly once
    for (int p = 0; p < pb.n_pat; ++p) {
      int64_t w = pb.w[p], r = pb.r[p], o = h % r;
      int64_t m = o >= w ? 0 : (w - o + r - 1) / r;
      for (int64_t seg = 0; seg * w < N; ++seg)
        for (int64_t k = 0; k < m; ++k) {
          const int64_t xk = seg * w + o + r * k;
          if (xk >= N) break;  // a last segment cut short by the sequence's end
          if (xk < pb.q0 || xk >= pb.q1) continue;  // outside the computed part
          auto it = seen.find(std::make_tuple(p, seg, k));
          CHECK(it != seen.end() && it->second == 1, "%s: row p=%d seg=%ld k=%ld seen %d times\n", name, p, (long)seg, (long)k, it == seen.end() ? 0 : it->second);
        }
    }
    for (int64_t x = 0; x < N; ++x) {
      bool covered = false;
      for (int p = 0; p < pb.n_pat; ++p) {
        int64_t w = pb.w[p], r = pb.r[p], o = h % r;
        int64_t rel = x - (x / w) * w - o;
        if (rel >= 0 && rel % r == 0) covered = true;
      }
      const bool in_part = x >= pb.q0 && x < pb.q1;
      CHECK(finalized[x] == (covered && in_part ? 1 : 0), "%s: position %ld finalized %d times (covered %d)\n", name, (long)x, finalized[x], covered);
      if (!covered) CHECK(P.uncovered_possible, "%s: uncovered position but flag off\n", name);
    }
  }
  if (!quiet || fails != f0)
    printf("%-28s ranges=%d units=%d R=%ld tiles/head=%.1f kv/head=%.1f %s\n", name, P.n_ranges, P.n_units,
           (long)P.range_len, (double)n_tiles / H, (double)n_kv / H, fails == f0 ? "OK" : "FAIL");
  return true;
}

// Seeded random shapes the kernel takes: N a multiple of 64 up to 16384,
// 1..6 patterns, w dividing N or (one in three) any length up to 1.5 N,
// r up to 16 (r > w allowed), 1..12 heads,
// causal or not, and SM counts that change the unit plan.
void random_cases(int count) {
  uint64_t st = 0x9e3779b97f4a7c15ull;
  auto next = [&]() { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; };
  const int64_t rs[] = {1, 1, 2, 3, 4, 5, 6, 7, 8, 12, 16};
  const int sms[] = {148, 132, 16, 1};
  int ran = 0, f0 = fails;
  for (int c = 0; c < count; ++c) {
    const int64_t N = 64 * (int64_t)(2 + next() % 255);
    std::vector<int64_t> divs;
    for (int64_t w = 2; w <= N; ++w)
      if (N % w == 0) divs.push_back(w);
    const int n_pat = 1 + (int)(next() % 6);
    std::vector<std::pair<int64_t, int64_t>> pats;
    for (int i = 0; i < n_pat; ++i) {
      // every third pattern: any w up to 1.5 N (a shorter last segment, or w > N)
      const int64_t w = next() % 3 == 0 ? 2 + (int64_t)(next() % (uint64_t)(N + N / 2)) : divs[next() % divs.size()];
      pats.push_back({w, rs[next() % (sizeof(rs) / sizeof(rs[0]))]});
    }
    const int64_t H = 1 + (int64_t)(next() % 12);
    const int causal = (int)(next() & 1);
    char name[64];
    snprintf(name, sizeof(name), "random%d", c);
    const int f1 = fails;
    if (!run_case(name, 1, N, H, pats, causal, sms[next() % 4], true)) continue;
    if (fails != f1) {
      printf("  N=%ld H=%ld causal=%d patterns:", (long)N, (long)H, causal);
      for (auto& pr : pats) printf(" (%ld,%ld)", (long)pr.first, (long)pr.second);
      printf("\n");
    }
    ++ran;
  }
  printf("random cases: %d of %d taken by the kernel, %s\n", ran, count, fails == f0 ? "OK" : "FAIL");
}

// Multiply-shift division against plain division: every divisor up to 4100
// with every dividend up to 70000, then random pairs over the whole range.
void check_fastdiv() {
  for (int d = 1; d <= 4100; ++d) {
    const FastDiv f = make_fastdiv(d);
    for (int x = 0; x < 70000; ++x)
      CHECK(fdiv(x, f) == x / d, "fdiv %d / %d\n", x, d);
  }
  uint64_t st = 88172645463325252ull;
  auto next = [&]() { st ^= st << 13; st ^= st >> 7; st ^= st << 17; return st; };
  for (int i = 0; i < 4000000; ++i) {
    const int64_t d = 1 + (int64_t)(next() % ((uint64_t)1 << (1 + next() % 30)));
    const int x = (int)(next() & 0x7fffffffu);
    CHECK(fdiv(x, make_fastdiv(d)) == (int)(x / d), "fdiv %d / %ld\n", x, (long)d);
  }
  for (int64_t d : {(int64_t)1, (int64_t)3, (int64_t)4095, (int64_t)4096, (int64_t)65537, ((int64_t)1 << 30) - 1, (int64_t)1 << 30}) {
    const FastDiv f = make_fastdiv(d);
    for (int x : {0, 1, (int)d - 1, (int)d, 0x7ffffffe, 0x7fffffff})
      if (x >= 0) CHECK(fdiv(x, f) == (int)(x / d), "fdiv edge %d / %ld\n", x, (long)d);
  }
  printf("fastdiv %s\n", fails ? "FAIL" : "OK");
}

int main() {
  check_fastdiv();
  run_case("lm", 1, 8192, 12, {{2048, 1}, {4096, 2}, {8192, 4}}, 1);
  run_case("long32k", 1, 32768, 12, {{2048, 1}, {4096, 2}, {8192, 4}, {16384, 6}, {32768, 12}}, 1);
  run_case("smallseg", 1, 8192, 8, {{64, 1}, {64, 2}}, 0);
  run_case("sweep64k", 1, 65536, 8, {{2048, 1}, {4096, 2}, {8192, 4}, {16384, 8}, {32768, 16}, {65536, 32}}, 1);
  run_case("lm_like", 1, 2048, 4, {{512, 1}, {1024, 2}, {2048, 4}}, 1);
  run_case("paper_like", 1, 3072, 6, {{256, 1}, {512, 2}, {1024, 4}, {1536, 6}, {3072, 12}}, 1);
  run_case("dup_unordered", 1, 1024, 3, {{1024, 4}, {256, 1}, {256, 1}}, 1);
  run_case("noncausal_small", 1, 1024, 4, {{64, 1}, {64, 2}}, 0);
  run_case("no_r1", 1, 1536, 5, {{384, 3}, {768, 4}, {1536, 8}}, 1);
  run_case("w_eq_N", 1, 640, 2, {{640, 1}}, 1);
  run_case("r_gt_w", 1, 512, 4, {{512, 1}, {2, 3}}, 1);
  run_case("odd_mix", 1, 6000, 7, {{600, 1}, {1200, 7}, {3000, 5}, {6000, 9}}, 1);
  run_case("odd_mix_nc", 1, 6000, 7, {{600, 1}, {1200, 7}, {3000, 5}, {6000, 9}}, 0);
  run_case("sweep1M_part", 1, 1048576, 1, {{2048, 1}, {4096, 2}, {8192, 4}, {16384, 8}, {32768, 16}, {65536, 32}}, 1);
  // computed parts: a sequence shard (positions), a head range, unaligned bounds
  run_case("long32k_shard1of2", 1, 32768, 12, {{2048, 1}, {4096, 2}, {8192, 4}, {16384, 6}, {32768, 12}}, 1, 148,
           false, 16384, 32768);
  run_case("long32k_shard3of4_heads", 1, 32768, 12, {{2048, 1}, {4096, 2}, {8192, 4}, {16384, 6}, {32768, 12}}, 1,
           148, false, 16384, 24576, 3, 9);
  run_case("lm_unaligned_part", 1, 8192, 12, {{2048, 1}, {4096, 2}, {8192, 4}}, 1, 148, false, 1000, 7001, 5, 6);
  run_case("noncausal_part", 1, 6000, 7, {{600, 1}, {1200, 7}, {3000, 5}, {6000, 9}}, 0, 132, false, 777, 4321, 1, 7);
  // partial last segments (w not dividing N) and w > N
  run_case("long32k_minus64", 1, 32704, 12, {{2048, 1}, {4096, 2}, {8192, 4}, {16384, 6}, {32768, 12}}, 1);
  run_case("long32k_minus64_nc", 1, 32704, 12, {{2048, 1}, {4096, 2}, {8192, 4}, {16384, 6}, {32768, 12}}, 0);
  run_case("partial_odd", 1, 5000, 5, {{768, 1}, {1536, 3}, {4096, 7}, {9000, 5}}, 1);
  run_case("partial_odd_nc", 1, 5000, 5, {{768, 1}, {1536, 3}, {4096, 7}, {9000, 5}}, 0);
  run_case("partial_777", 1, 777, 2, {{128, 1}, {256, 4}}, 1);
  run_case("partial_1000_nc", 2, 1000, 4, {{256, 1}, {384, 2}}, 0);
  run_case("partial_part", 1, 10000, 6, {{3000, 1}, {7000, 3}}, 0, 148, false, 2999, 9001, 2, 5);
  random_cases(300);
  printf("fails=%d\n", fails);
  return fails ? 1 : 0;
}
