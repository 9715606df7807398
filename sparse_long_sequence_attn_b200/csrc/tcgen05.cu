// Kernel family TCGEN05: fused multi-pattern dilated flash-attention forward
// for bf16, D = 64, on the 5th-generation tensor cores of sm_100a.
//
// What it computes ("LONGNET: Scaling Transformer to 1 billion tokens",
// section "LongNet's attention allocation principle"; "LongNet论文精读",
// section "Dilated Attention的工作原理"): for every pattern (w, r), segments of
// w tokens, head h keeping the rows o + r*k < w (o = h mod r), causal or full
// softmax(Q K^T / sqrt(D)) V on each sparsified segment, rows put back at
// their positions, and the patterns combined per row with weights equal to
// their softmax denominators.
//
// Design.
//  * Work unit = (batch b, head h, position range [A, A + R)), R = 128 * r_max.
//    One CTA per unit; units are launched longest-first (host cost model), so
//    the hardware block scheduler does greedy LPT balancing.
//  * Inside a unit, every pattern's kept rows are cut into "natural" tiles of
//    up to 128 consecutive kept rows of one segment (clipped to the range), so
//    each tile is a dense block of a w/r x w/r attention problem: no MMA rows
//    are wasted on rows of other patterns.
//  * Dilated gather: one 5-D TMA tensor map per distinct r views [B, N, H, D]
//    as (d, h, c, k, b) with position = r*k + c, so a box of 128 consecutive
//    k at fixed (c, h, b) is exactly 128 kept rows, 128 B each, landing in
//    shared memory with the 128-byte swizzle the tensor cores read.  A second
//    map per r, shifted by N mod r positions, reaches the last few rows.
//  * S = Q K^T and O += P V run as tcgen05.mma (bf16 in, fp32 accumulate in
//    tensor memory).  S is double-buffered in TMEM; P (bf16) overwrites the
//    first half of its S buffer and is read from TMEM by the PV MMA.
//  * Online softmax in fp32 by one warpgroup (thread i owns row i), exp2 on
//    scaled scores, lazy rescaling of O (only when the row max grows by more
//    than 2^8).
//  * Cross-pattern combination without any HBM round trip: tiles are
//    processed in order of (first position, larger r first, pattern index).
//    Each tile's epilogue decides per row whether it is the last tile
//    covering that position; if not, it parks the normalised row (bf16) and
//    its lse in a per-pattern shared-memory slot; the last one merges the
//    parked rows of the other patterns and writes `out` / `lse` once.  With
//    this order a pattern's slot is always fully consumed before that pattern's
//    next tile overwrites it, so one 16 KB slot per pattern is enough.
//  * Every wait is bounded; on a timeout the kernel records the status word,
//    stops issuing work, drains what it issued and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <numeric>
#include <vector>

#include "device_util.cuh"
#include "params.h"

namespace longnet {
namespace tc {

constexpr int kD = 64;          // head dimension of this family
constexpr int kBM = 128;        // query rows per tile (MMA M)
constexpr int kBN = 128;        // keys per KV block (MMA N of Q K^T)
constexpr int kStages = 3;      // K/V shared-memory ring depth
constexpr int kMaxPat = 6;      // patterns (and combination slots) supported
constexpr int kMaxR = 8;        // distinct dilations supported
constexpr int kThreads = 256;   // 8 warps: TMA, MMA, 2 idle, 4 softmax/epilogue
constexpr int kTileBytes = kBM * kD * 2;  // 16 KB per 128 x 64 bf16 tile
constexpr int kMaxRangeOrder = 4096;

// TMEM columns: two S buffers (128 fp32 columns each) and O (64 columns).
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;

struct SmemLayout {
  static constexpr int q = 0;
  static constexpr int k = q + kTileBytes;
  static constexpr int v = k + kStages * kTileBytes;
  static constexpr int slot_o = v + kStages * kTileBytes;
  static constexpr int slot_l = slot_o + kMaxPat * kTileBytes;
  static constexpr int bars = slot_l + kMaxPat * kBM * 4;
  static constexpr int n_bars = 2 + 2 * kStages + 2 + 2 + 3;
  static constexpr int misc = bars + n_bars * 8;
  static constexpr int total = misc + 64;
};
constexpr int kSmemBytes = SmemLayout::total + 1024;  // + alignment slack

struct __align__(64) TmaMaps {
  CUtensorMap m[kMaxR][2][3];  // [distinct r][base / shifted][q, k, v]
};

struct Params {
  Problem pb;
  int n_r;                    // distinct dilations
  int r_val[kMaxR];           // their values
  int tail[kMaxR];            // N mod r
  int kfull[kMaxR];           // N div r
  int pat_r[kMaxPat];         // index into r_val of each pattern
  int range_len;              // R
  int n_ranges;
  int uncovered_possible;     // some position may be kept by no pattern
  uint64_t wait_limit_ns;
  int range_order[kMaxRangeOrder];  // longest-first order of ranges (or -1: identity)
};

// ---------------------------------------------------------------- PTX bits

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
      "r"(c4)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

#define LN_TMEM_LD32(taddr, r)                                                                  \
  asm volatile(                                                                                 \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13," \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"       \
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),     \
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),              \
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),           \
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),           \
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),           \
        "=r"(r[31])                                                                             \
      : "r"(taddr))

#define LN_TMEM_ST32(taddr, r)                                                                 \
  asm volatile(                                                                                \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12," \
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"     \
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]),          \
        "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]),        \
        "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]),    \
        "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]),    \
        "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]))

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 version field.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t addr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // SWIZZLE_128B
  return d;
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> fp32, given M, N, B major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4)                      // D format: f32
         | (1u << 7)                    // A format: bf16
         | (1u << 10)                   // B format: bf16
         | ((b_mn_major ? 1u : 0u) << 16)
         | ((uint32_t)(N >> 3) << 17)   // N / 8
         | ((uint32_t)(M >> 4) << 24);  // M / 16
}
constexpr uint32_t kIdescQK = idesc_bf16(kBM, kBN, false);
constexpr uint32_t kIdescPV = idesc_bf16(kBM, kD, true);

// ---------------------------------------------------------------- tiles

struct Tile {
  int p;          // pattern index
  int seg;    // segment index
  int k0;     // first kept row (sparse index within the segment)
  int nrows;      // rows in this tile (<= 128)
  int nkv;        // KV blocks of 128 keys
  int start;  // position of the first row
};

// Walks the unit's tiles in processing order.  All roles run identical copies.
struct TileWalker {
  int n_pat;
  int A, Bnd;  // range [A, Bnd)
  int w[kMaxPat], r[kMaxPat], o[kMaxPat], m[kMaxPat];
  int seg[kMaxPat], k0[kMaxPat], khi[kMaxPat], seg_last[kMaxPat];
  bool causal;

  __host__ __device__ void seg_bounds(int p) {
    // kept rows of segment seg[p] whose positions fall in [A, Bnd)
    const int base = seg[p] * w[p] + o[p];
    int lo = A - base;
    lo = lo <= 0 ? 0 : (lo + r[p] - 1) / r[p];
    int hi = Bnd - base;
    hi = hi <= 0 ? 0 : (hi + r[p] - 1) / r[p];
    if (hi > m[p]) hi = m[p];
    k0[p] = lo;
    khi[p] = hi;
  }
  __host__ __device__ void advance_to_nonempty(int p) {
    while (seg[p] <= seg_last[p] && k0[p] >= khi[p]) {
      ++seg[p];
      if (seg[p] <= seg_last[p]) seg_bounds(p);
    }
  }
  __host__ __device__ void init(const Params& P, int h, int a, int bnd) {
    n_pat = P.pb.n_pat;
    A = a;
    Bnd = bnd;
    causal = P.pb.causal != 0;
    for (int p = 0; p < n_pat; ++p) {
      w[p] = P.pb.w[p];
      r[p] = P.pb.r[p];
      o[p] = h % r[p];
      m[p] = o[p] >= w[p] ? 0 : (w[p] - o[p] + r[p] - 1) / r[p];
      seg[p] = A / w[p];
      seg_last[p] = (Bnd - 1) / w[p];
      seg_bounds(p);
      advance_to_nonempty(p);
    }
  }
  __host__ __device__ bool next(Tile& t) {
    int best = -1;
    int best_start = 0;
    for (int p = 0; p < n_pat; ++p) {
      if (seg[p] > seg_last[p]) continue;
      const int st = seg[p] * w[p] + o[p] + r[p] * k0[p];
      if (best < 0 || st < best_start || (st == best_start && r[p] > r[best])) {
        best = p;
        best_start = st;
      }
    }
    if (best < 0) return false;
    const int p = best;
    t.p = p;
    t.seg = seg[p];
    t.k0 = k0[p];
    const int n = khi[p] - k0[p];
    t.nrows = (int)(n < kBM ? n : kBM);
    t.start = best_start;
    const int nkeys = causal ? k0[p] + t.nrows : m[p];
    t.nkv = (int)((nkeys + kBN - 1) / kBN);
    k0[p] += t.nrows;
    advance_to_nonempty(p);
    return true;
  }
};

// Processing-order key of the tile of pattern q that covers position x in
// the unit [A, Bnd); returns false when q does not keep x.
struct Cover {
  int start;
  int slot_row;
};
__host__ __device__ inline bool cover_of(const TileWalker& tw, int q, int x, Cover& c) {
  const int sq = x / tw.w[q];
  const int rel = x - sq * tw.w[q] - tw.o[q];
  if (rel < 0) return false;
  const int kq = rel / tw.r[q];
  if (kq * tw.r[q] != rel) return false;
  if (kq >= tw.m[q]) return false;
  const int base = sq * tw.w[q] + tw.o[q];
  int lo = tw.A - base;
  lo = lo <= 0 ? 0 : (lo + tw.r[q] - 1) / tw.r[q];
  const int t = (kq - lo) / kBM;
  c.start = base + tw.r[q] * (lo + t * kBM);
  c.slot_row = (int)((kq - lo) - t * kBM);
  return true;
}
__host__ __device__ inline bool key_before(int s_a, int r_a, int p_a, int s_b,
                                           int r_b, int p_b) {
  if (s_a != s_b) return s_a < s_b;
  if (r_a != r_b) return r_a > r_b;
  return p_a < p_b;
}

// ---------------------------------------------------------------- waits

struct Sync {
  uint64_t* bars;
  volatile int* abort_flag;
  int* status;
  uint64_t limit;
  // All lanes wait; the warp proceeds only if every lane saw the phase, so
  // warp-collective tcgen05 instructions stay convergent on every path.
  __device__ bool wait_warp(uint64_t* bar, uint32_t parity) {
    const bool ok = wait(bar, parity);
    return __all_sync(0xffffffffu, ok);
  }
  __device__ bool wait(uint64_t* bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t it = 1;; ++it) {
      if (mbar_try_wait(a, parity)) return true;
      if ((it & 15u) == 0) {
        if (*abort_flag) return false;
        if (global_ns() - t0 > limit) {
          *abort_flag = 1;
          record_status(status, kStatusTimeout);
          return false;
        }
      }
    }
  }
};

// TMA coordinates of 128 kept rows starting at sparse row k of pattern p,
// segment seg, head h, batch b.  `need` = kept rows that must be real data.
struct TmaCoord {
  int map;  // 0 base map, 1 shifted map
  int c, kk;
};
__host__ __device__ inline TmaCoord tma_coord(const Params& P, int ri, int first_pos,
                                              int need) {
  const int r = P.r_val[ri];
  const int last_pos = first_pos + r * (need - 1);
  TmaCoord t;
  if (last_pos >= r * P.kfull[ri]) {
    const int x = first_pos - P.tail[ri];  // >= 0 by the host's shape check
    t.map = 1;
    t.c = (int)(x % r);
    t.kk = (int)(x / r);
  } else {
    t.map = 0;
    t.c = (int)(first_pos % r);
    t.kk = (int)(first_pos / r);
  }
  return t;
}

// ---------------------------------------------------------------- kernel

__global__ void __launch_bounds__(kThreads, 1)
    dilated_fwd_kernel(const __grid_constant__ Params P, const __grid_constant__ TmaMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + SmemLayout::q;
  uint8_t* sK = smem + SmemLayout::k;
  uint8_t* sV = smem + SmemLayout::v;
  uint8_t* sSlotO = smem + SmemLayout::slot_o;
  float* sSlotL = reinterpret_cast<float*>(smem + SmemLayout::slot_l);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SmemLayout::bars);
  uint64_t* bar_q_full = bars + 0;
  uint64_t* bar_q_empty = bars + 1;
  uint64_t* bar_kv_full = bars + 2;
  uint64_t* bar_kv_empty = bars + 2 + kStages;
  uint64_t* bar_s_full = bars + 2 + 2 * kStages;
  uint64_t* bar_p_full = bar_s_full + 2;
  uint64_t* bar_o_done = bar_p_full + 2;
  uint64_t* bar_o_free = bar_o_done + 1;
  uint64_t* bar_drain = bar_o_free + 1;
  uint64_t* bar_epi = bar_drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + SmemLayout::misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + SmemLayout::misc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // unit -> (b, h, range)
  const int64_t BH = P.pb.B * P.pb.H;
  const int64_t rank = blockIdx.x / BH;
  const int64_t bh = blockIdx.x - rank * BH;
  const int64_t b = bh / P.pb.H;
  const int64_t h = bh - b * P.pb.H;
  const int ri_range = (P.range_order[0] >= 0 && rank < kMaxRangeOrder) ? P.range_order[rank] : (int)rank;
  const int A = ri_range * P.range_len;
  const int Bnd = (int64_t)A + P.range_len < P.pb.N ? A + P.range_len : (int)P.pb.N;

  if (threadIdx.x == 0) {
    mbar_init(bar_q_full, 1);
    mbar_init(bar_q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_kv_full + s, 1);
      mbar_init(bar_kv_empty + s, 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar_s_full + s, 1);
      mbar_init(bar_p_full + s, 128);
    }
    mbar_init(bar_o_done, 1);
    mbar_init(bar_o_free, 128);
    mbar_init(bar_drain, 1);
    mbar_init(bar_epi, 128);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < P.n_r; ++i)
      for (int j = 0; j < 2; ++j)
        for (int t = 0; t < 3; ++t) prefetch_tmap(&maps.m[i][j][t]);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  Sync sy{bars, abort_flag, P.pb.status, P.wait_limit_ns};
  TileWalker tw;
  tw.init(P, h, A, Bnd);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t kv_it = 0, tile_it = 0;
      Tile t;
      bool ok = true;
      while (ok && tw.next(t)) {
        const int ri = P.pat_r[t.p];
        const int seg_base = t.seg * tw.w[t.p] + tw.o[t.p];
        if (tile_it > 0) ok = sy.wait(bar_q_empty, (tile_it - 1) & 1);
        if (!ok) break;
        {
          const int first = seg_base + tw.r[t.p] * t.k0;
          const TmaCoord c = tma_coord(P, ri, first, t.nrows);
          mbar_arrive_expect_tx(bar_q_full, kTileBytes);
          tma_load_5d(sQ, &maps.m[ri][c.map][0], bar_q_full, 0, (int)h, c.c, c.kk, (int)b);
        }
        const int n_keys_total = tw.causal ? t.k0 + t.nrows : tw.m[t.p];
        for (int j = 0; j < t.nkv; ++j) {
          const int s = kv_it % kStages;
          if (kv_it >= kStages) ok = sy.wait(bar_kv_empty + s, ((kv_it / kStages) - 1) & 1);
          if (!ok) break;
          const int kstart = j * kBN;
          int need = n_keys_total - kstart;
          if (need > kBN) need = kBN;
          const int first = seg_base + tw.r[t.p] * kstart;
          const TmaCoord c = tma_coord(P, ri, first, need);
          mbar_arrive_expect_tx(bar_kv_full + s, 2 * kTileBytes);
          tma_load_5d(sK + s * kTileBytes, &maps.m[ri][c.map][1], bar_kv_full + s, 0, (int)h, c.c,
                      c.kk, (int)b);
          tma_load_5d(sV + s * kTileBytes, &maps.m[ri][c.map][2], bar_kv_full + s, 0, (int)h, c.c,
                      c.kk, (int)b);
          ++kv_it;
        }
        ++tile_it;
      }
      // drain: every issued K/V load has landed before the CTA may exit
      for (uint32_t i = (kv_it > kStages ? kv_it - kStages : 0); i < kv_it; ++i) {
        const int s = i % kStages;
        if (!mbar_wait(bar_kv_full + s, (i / kStages) & 1, P.wait_limit_ns)) {
          record_status(P.pb.status, kStatusTimeout);
          break;
        }
      }
      if (tile_it > 0) {
        if (!mbar_wait(bar_q_full, (tile_it - 1) & 1, P.wait_limit_ns))
          record_status(P.pb.status, kStatusTimeout);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ);
      uint32_t kv_it = 0, tile_it = 0, s_it = 0;
      Tile t;
      bool ok = true;
      while (ok && tw.next(t)) {
        ok = sy.wait(bar_q_full, tile_it & 1);
        if (!ok) break;
        tc_fence_after();
        int pend_stage = -1;
        uint32_t pend_s = 0;
        bool pend_first = false;
        for (int j = 0; j <= t.nkv && ok; ++j) {
          if (j < t.nkv) {
            const int st = kv_it % kStages;
            ok = sy.wait(bar_kv_full + st, (kv_it / kStages) & 1);
            if (!ok) break;
            tc_fence_after();
            const uint32_t sb = s_it & 1;
            const uint32_t d = tmem + (sb ? kColS1 : kColS0);
            const uint32_t k_addr = smem_u32(sK + st * kTileBytes);
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
              const uint64_t ad = smem_desc_sw128(q_addr + kk * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(k_addr + kk * 32, 16, 1024);
              mma_ss(d, ad, bd, kIdescQK, kk > 0 ? 1u : 0u);
            }
            tc_commit(bar_s_full + sb);
            if (j == t.nkv - 1) tc_commit(bar_q_empty);
          }
          if (pend_stage >= 0) {
            // O += P V for the previous block
            const uint32_t sb = pend_s & 1;
            ok = sy.wait(bar_p_full + sb, (pend_s >> 1) & 1);
            if (!ok) break;
            if (pend_first && tile_it > 0) {
              ok = sy.wait(bar_o_free, (tile_it - 1) & 1);
              if (!ok) break;
            }
            tc_fence_after();
            const uint32_t v_addr = smem_u32(sV + pend_stage * kTileBytes);
            const uint32_t p_tmem = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              const uint64_t bd = smem_desc_sw128(v_addr + kk * 2048, kBN * 128, 1024);
              mma_ts(tmem + kColO, p_tmem + kk * 8, bd, kIdescPV,
                     (pend_first && kk == 0) ? 0u : 1u);
            }
            tc_commit(bar_kv_empty + pend_stage);
            tc_commit(bar_o_done);
            pend_stage = -1;
          }
          if (j < t.nkv) {
            pend_stage = kv_it % kStages;
            pend_s = s_it;
            pend_first = (j == 0);
            ++kv_it;
            ++s_it;
          }
        }
        ++tile_it;
      }
      // drain: all issued MMAs complete before TMEM is released
      tc_commit(bar_drain);
      if (!mbar_wait(bar_drain, 0, P.wait_limit_ns)) record_status(P.pb.status, kStatusTimeout);
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax + epilogue
    const int row = (warp - 4) * 32 + lane;
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)kD);
    uint32_t s_it = 0, tile_it = 0;
    Tile t;
    bool ok = true;
    __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(P.pb.out);
    while (ok && tw.next(t)) {
      float m_use = -INFINITY, l_run = 0.f;
      const int krow = t.k0 + row;  // this thread's sparse row
      for (int j = 0; j < t.nkv; ++j) {
        const uint32_t sb = s_it & 1;
        ok = sy.wait_warp(bar_s_full + sb, (s_it >> 1) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_col = tmem + lane_base + (sb ? kColS1 : kColS0);
        uint32_t sr[kBN];
        // four loads in flight, one wait
        LN_TMEM_LD32(s_col + 0, (sr + 0));
        LN_TMEM_LD32(s_col + 32, (sr + 32));
        LN_TMEM_LD32(s_col + 64, (sr + 64));
        LN_TMEM_LD32(s_col + 96, (sr + 96));
        tmem_wait_ld();
        float s[kBN];
#pragma unroll
        for (int c = 0; c < kBN; ++c) s[c] = __uint_as_float(sr[c]);
        // masks: causal (key <= row) and keys past the segment's kept rows
        const int kbase = j * kBN;
        const int lim = tw.causal ? krow - kbase : tw.m[t.p] - 1 - kbase;
        if (lim < kBN - 1) {
#pragma unroll
          for (int c = 0; c < kBN; ++c)
            if (c > lim) s[c] = -INFINITY;
        }
        // row max as a tree (independent partial maxima)
        float pm[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) pm[e] = s[e];
#pragma unroll
        for (int c = 8; c < kBN; c += 8)
#pragma unroll
          for (int e = 0; e < 8; ++e) pm[e] = fmaxf(pm[e], s[c + e]);
        const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                               fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        const float m_blk = mx * scale_log2;
        float corr = 1.f;
        bool rescale = false;
        if (m_blk > m_use + 8.f || m_use == -INFINITY) {
          if (m_blk != -INFINITY) {
            if (m_use != -INFINITY) {
              corr = ex2(m_use - m_blk);
              rescale = true;
            }
            m_use = m_blk;
          }
        }
        float ps[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) ps[e] = 0.f;
        const uint32_t p_col = s_col;  // P overwrites the first 64 columns of S
#pragma unroll
        for (int c = 0; c < kBN / 64; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float a = ex2(fmaf(s[c * 64 + 2 * e], scale_log2, -m_use));
            const float bq = ex2(fmaf(s[c * 64 + 2 * e + 1], scale_log2, -m_use));
            ps[e & 7] += a + bq;
            pk[e] = pack_bf16(a, bq);
          }
          LN_TMEM_ST32(p_col + c * 32, pk);
        }
        const float lsum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        tmem_wait_st();
        l_run = l_run * corr + lsum;
        if (j > 0) {
          // PV of the previous block must be done before O is touched
          ok = sy.wait_warp(bar_o_done, (s_it - 1) & 1);
          if (!ok) break;
          tc_fence_after();
          if (__any_sync(0xffffffffu, rescale)) {
            const uint32_t o_col = tmem + lane_base + kColO;
            uint32_t rr[kD];
            LN_TMEM_LD32(o_col, (rr + 0));
            LN_TMEM_LD32(o_col + 32, (rr + 32));
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < kD; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * corr);
            LN_TMEM_ST32(o_col, (rr + 0));
            LN_TMEM_ST32(o_col + 32, (rr + 32));
            tmem_wait_st();
          }
        }
        tc_fence_before();
        mbar_arrive(bar_p_full + sb);
        ++s_it;
      }
      if (!ok) break;
      // ---- epilogue of this tile
      ok = sy.wait_warp(bar_o_done, (s_it - 1) & 1);
      if (!ok) break;
      tc_fence_after();
      float o[kD];
      {
        const uint32_t o_col = tmem + lane_base + kColO;
        uint32_t rr[kD];
        LN_TMEM_LD32(o_col, (rr + 0));
        LN_TMEM_LD32(o_col + 32, (rr + 32));
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < kD; ++e) o[e] = __uint_as_float(rr[e]);
      }
      tc_fence_before();
      mbar_arrive(bar_o_free);
      if (row < t.nrows) {
        const float inv = 1.f / l_run;
#pragma unroll
        for (int d = 0; d < kD; ++d) o[d] *= inv;
        float lse2 = m_use + __log2f(l_run);  // log2 domain
        const int x = t.start + tw.r[t.p] * row;
        // last tile covering x?  (all other covering tiles come earlier)
        bool final_row = true;
        for (int q = 0; q < tw.n_pat && final_row; ++q) {
          if (q == t.p) continue;
          Cover cv;
          if (!cover_of(tw, q, x, cv)) continue;
          if (!key_before(cv.start, tw.r[q], q, t.start, tw.r[t.p], t.p)) final_row = false;
        }
        if (final_row) {
          for (int q = 0; q < tw.n_pat; ++q) {
            if (q == t.p) continue;
            Cover cv;
            if (!cover_of(tw, q, x, cv)) continue;
            const float lq = sSlotL[q * kBM + cv.slot_row];
            const float mxl = fmaxf(lse2, lq);
            const float wa = ex2(lse2 - mxl), wb = ex2(lq - mxl);
            const float inv2 = 1.f / (wa + wb);
            const uint4* src = reinterpret_cast<const uint4*>(sSlotO + q * kTileBytes + cv.slot_row * 128);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
              const uint4 u = src[ch ^ (cv.slot_row & 7)];
              const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat162 pr = *reinterpret_cast<const __nv_bfloat162*>(&wv[e]);
                const int d = ch * 8 + e * 2;
                o[d] = (wa * o[d] + wb * __bfloat162float(pr.x)) * inv2;
                o[d + 1] = (wa * o[d + 1] + wb * __bfloat162float(pr.y)) * inv2;
              }
            }
            lse2 = mxl + __log2f(wa + wb);
          }
          uint4* dst = reinterpret_cast<uint4*>(outp + ((b * P.pb.N + x) * P.pb.H + h) * kD);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint4 u;
            u.x = pack_bf16(o[ch * 8 + 0], o[ch * 8 + 1]);
            u.y = pack_bf16(o[ch * 8 + 2], o[ch * 8 + 3]);
            u.z = pack_bf16(o[ch * 8 + 4], o[ch * 8 + 5]);
            u.w = pack_bf16(o[ch * 8 + 6], o[ch * 8 + 7]);
            dst[ch] = u;
          }
          if (P.pb.lse) P.pb.lse[(b * P.pb.H + h) * P.pb.N + x] = lse2 * 0.69314718055994531f;
        } else {
          uint4* dst = reinterpret_cast<uint4*>(sSlotO + t.p * kTileBytes + row * 128);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            uint4 u;
            u.x = pack_bf16(o[ch * 8 + 0], o[ch * 8 + 1]);
            u.y = pack_bf16(o[ch * 8 + 2], o[ch * 8 + 3]);
            u.z = pack_bf16(o[ch * 8 + 4], o[ch * 8 + 5]);
            u.w = pack_bf16(o[ch * 8 + 6], o[ch * 8 + 7]);
            dst[ch ^ (row & 7)] = u;
          }
          sSlotL[t.p * kBM + row] = lse2;
        }
      }
      // parked rows become visible to the next epilogue's threads (a bounded
      // barrier of the 128 softmax threads)
      mbar_arrive(bar_epi);
      ok = sy.wait_warp(bar_epi, tile_it & 1);
      ++tile_it;
    }
    if (ok && P.uncovered_possible) {
      // positions of this range that no pattern keeps: out = 0, lse = -inf
      for (int x = A + row; x < Bnd; x += 128) {
        bool any = false;
        for (int q = 0; q < tw.n_pat && !any; ++q) {
          Cover cv;
          any = cover_of(tw, q, x, cv);
        }
        if (!any) {
          uint4* dst = reinterpret_cast<uint4*>(outp + ((b * P.pb.N + x) * P.pb.H + h) * kD);
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) dst[ch] = make_uint4(0, 0, 0, 0);
          if (P.pb.lse) P.pb.lse[(b * P.pb.H + h) * P.pb.N + x] = -INFINITY;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

// View [B, N, H, D] bf16 (starting `shift` positions in) as (d, h, c, k, b)
// with position = shift + r*k + c, k < kcount.
bool encode_map(EncodeTiledFn enc, CUtensorMap* map, const void* base, const Problem& p, int64_t r,
                int64_t shift, int64_t kcount) {
  const int64_t es = 2;
  const char* ptr = static_cast<const char*>(base) + shift * p.H * kD * es;
  cuuint64_t dims[5] = {(cuuint64_t)kD, (cuuint64_t)p.H, (cuuint64_t)r, (cuuint64_t)kcount,
                        (cuuint64_t)p.B};
  cuuint64_t strides[4] = {(cuuint64_t)(kD * es), (cuuint64_t)(p.H * kD * es),
                           (cuuint64_t)(r * p.H * kD * es), (cuuint64_t)(p.N * p.H * kD * es)};
  cuuint32_t box[5] = {(cuuint32_t)kD, 1, 1, (cuuint32_t)kBM, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult rc = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<char*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return rc == CUDA_SUCCESS;
}

int64_t r_max_of(const Problem& p) {
  int64_t rm = 1;
  for (int i = 0; i < p.n_pat; ++i) rm = std::max(rm, p.r[i]);
  return rm;
}

// Host copy of the tile walk (same arithmetic) for the cost model.
int64_t range_cost(const Problem& pb, int64_t A, int64_t Bnd) {
  int64_t cost = 0;
  for (int p = 0; p < pb.n_pat; ++p) {
    const int64_t w = pb.w[p], r = pb.r[p], o = 0;
    const int64_t m = (w - o + r - 1) / r;
    for (int64_t seg = A / w; seg <= (Bnd - 1) / w; ++seg) {
      const int64_t base = seg * w + o;
      int64_t lo = A - base;
      lo = lo <= 0 ? 0 : (lo + r - 1) / r;
      int64_t hi = Bnd - base;
      hi = hi <= 0 ? 0 : (hi + r - 1) / r;
      hi = std::min(hi, m);
      for (int64_t k0 = lo; k0 < hi; k0 += kBM) {
        const int64_t n = std::min<int64_t>(kBM, hi - k0);
        const int64_t keys = pb.causal ? k0 + n : m;
        cost += (keys + kBN - 1) / kBN + 2;  // + per-tile overhead
      }
    }
  }
  return cost;
}

}  // namespace tc

bool tcgen05_supports(const Problem& p) {
  using namespace tc;
  if (p.dtype != LONGNET_DTYPE_BF16 || p.D != kD) return false;
  if (p.n_pat > kMaxPat) return false;
  if (p.H > 65535 || p.B > 65535) return false;
  int n_r = 0;
  int64_t rv[kMaxR];
  for (int i = 0; i < p.n_pat; ++i) {
    bool found = false;
    for (int j = 0; j < n_r; ++j) found |= (rv[j] == p.r[i]);
    if (!found) {
      if (n_r == kMaxR) return false;
      rv[n_r++] = p.r[i];
    }
    const int64_t r = p.r[i];
    if (r > 4096) return false;
    const int64_t t = p.N % r;
    // a 128-row box must never need both the first t and the last t positions
    if (t > 0 && p.N < kBM * r + 2 * t) return false;
    if (p.N / r < 1) return false;
  }
  const int64_t R = kBM * r_max_of(p);
  const int64_t n_ranges = (p.N + R - 1) / R;
  if (n_ranges * p.B * p.H > 0x7fffffffLL) return false;
  return true;
}

// Host half of the launch: everything in Params but the tensor maps.
void fill_params(const Problem& pb, tc::Params& P) {
  using namespace tc;
  memset(&P, 0, sizeof(P));
  P.pb = pb;
  P.wait_limit_ns = kWaitLimitNs;
  for (int i = 0; i < pb.n_pat; ++i) {
    int j = 0;
    while (j < P.n_r && P.r_val[j] != pb.r[i]) ++j;
    if (j == P.n_r) {
      P.r_val[j] = pb.r[i];
      P.tail[j] = pb.N % pb.r[i];
      P.kfull[j] = pb.N / pb.r[i];
      ++P.n_r;
    }
    P.pat_r[i] = j;
  }
  bool has_r1 = false;
  for (int i = 0; i < pb.n_pat; ++i) has_r1 |= (pb.r[i] == 1);
  P.uncovered_possible = has_r1 ? 0 : 1;
  P.range_len = kBM * r_max_of(pb);
  P.n_ranges = (int)((pb.N + P.range_len - 1) / P.range_len);
  if (P.n_ranges <= kMaxRangeOrder) {
    std::vector<int64_t> cost(P.n_ranges);
    for (int i = 0; i < P.n_ranges; ++i)
      cost[i] = range_cost(pb, (int64_t)i * P.range_len, std::min<int64_t>(pb.N, (int64_t)(i + 1) * P.range_len));
    std::vector<int> idx(P.n_ranges);
    std::iota(idx.begin(), idx.end(), 0);
    std::stable_sort(idx.begin(), idx.end(), [&](int a, int c) { return cost[a] > cost[c]; });
    for (int i = 0; i < P.n_ranges; ++i) P.range_order[i] = idx[i];
  } else {
    P.range_order[0] = -1;
  }
}

int launch_tcgen05(const Problem& pb, cudaStream_t stream) {
  using namespace tc;
  EncodeTiledFn enc = get_encoder();
  if (!enc) return LONGNET_ERR_CUDA;
  static Params P;  // large; filled under a lock, copied into the launch
  static TmaMaps maps;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  fill_params(pb, P);
  const void* bases[3] = {pb.q, pb.k, pb.v};
  for (int i = 0; i < P.n_r; ++i) {
    for (int t = 0; t < 3; ++t) {
      if (!encode_map(enc, &maps.m[i][0][t], bases[t], pb, P.r_val[i], 0, P.kfull[i]))
        return LONGNET_ERR_CUDA;
      if (!encode_map(enc, &maps.m[i][1][t], bases[t], pb, P.r_val[i], P.tail[i], P.kfull[i]))
        return LONGNET_ERR_CUDA;
    }
  }
  static bool attr_set[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return LONGNET_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(dilated_fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kSmemBytes) != cudaSuccess)
      return LONGNET_ERR_CUDA;
    attr_set[dev] = true;
  }
  const int64_t grid = (int64_t)P.n_ranges * pb.B * pb.H;
  dilated_fwd_kernel<<<(unsigned)grid, kThreads, kSmemBytes, stream>>>(P, maps);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

}  // namespace longnet
