// Kernel family TCGEN05 backward: dq, dk, dv of the multi-pattern dilated
// attention forward for bf16 or fp16, D = 64, on the 5th-generation tensor
// cores of sm_100a.
//
// What it computes.  The forward combines the patterns of a row with weights
// equal to their softmax denominators ("LONGNET: Scaling Transformer to 1
// billion tokens", section "Token expansion reaches 1 billion+"), which is one
// softmax over every (pattern, key) pair reaching the row; its gradient is
// that of a single softmax over the same pairs.  With P_ij = e^{s_ij / sqrt(D)
// - lse_i} (lse_i the combined lse the forward saved), delta_i =
// <dout_i, out_i> and dS_ij = P_ij (<dout_i, v_j> - delta_i):
//   dq_i = sum_j dS_ij k_j / sqrt(D),  dk_j = sum_i dS_ij q_i / sqrt(D),
//   dv_j = sum_i P_ij dout_i,
// summed over the pairs (i, j) of every pattern keeping both rows.  The model
// is trained ("LONGNET: Scaling Transformer to 1 billion tokens", section
// "Distributed training"), so this is the step after the forward.
//
// Design.
//  * Work is cut per pattern, batch, head and segment (a "unit": the
//    sparsified segment of that pattern, kept row t at position
//    first + r t), and per 128-row tile of it: one CTA per (unit, tile), the
//    tiles of a unit launched together (longest first) so the blocks they
//    all stream are read from L2.
//  * Two kernels, so no tile pair needs atomics:
//      key-centric (dk, dv): the CTA holds a tile of 128 keys (K, V) and
//      streams 64-query blocks (Q, dout, lse, delta) through a 3-stage ring:
//        S^T = K Q^T and dP^T = V dout^T (tcgen05.mma, smem x smem -> TMEM),
//        P^T, dS^T by the compute warps, written back over S^T and dP^T in
//        the input format, then dV += P^T dout and dK += dS^T Q
//        (tcgen05.mma with A read from TMEM);
//      query-centric (dq): the CTA holds 128 queries (Q, dout) and streams
//        64-key blocks (K, V): S = Q K^T, dP = dout V^T, dS, dQ += dS K.
//    Every operand tile lands in shared memory through the dilated 5-D TMA
//    maps of the forward (position = r k + c, 128-byte swizzle), so the
//    dilated gather costs nothing; Q and dout serve both as K-major operands
//    of the score products and as MN-major operands of the gradient products.
//  * Roles: warp 0 loads (one lane issues the TMA; the warp gathers lse and
//    delta of the streamed queries), warp 1 issues the MMAs, warps 2-5 (one
//    thread per TMEM lane, i.e. per tile row) compute P and dS and run the
//    epilogue.  256 TMEM columns and about 83 KB of shared memory per CTA, so
//    two CTAs share an SM and one's MMAs overlap the other's softmax.
//  * A row kept by several patterns receives one fp32 atomic add per pattern
//    (at the end of the owning CTA); the call zeroes the gradients first.
//    delta_i is computed once per row by a small pass into the dq buffer
//    (which the dq kernel then overwrites), so the library still allocates
//    nothing.
//  * Every wait is bounded; on a timeout the kernel records the status word,
//    stops issuing, drains what it issued and returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "device_util.cuh"
#include "params.h"
#include "tc_ptx.cuh"

namespace longnet {
namespace tb {
using namespace tc;

constexpr int kTile = 128;                      // rows a CTA owns (M of every MMA)
constexpr int kBlk = 64;                        // rows of a streamed block (N of the score MMAs)
constexpr int kMaxPat = 6;
constexpr int kStages = 3;
constexpr int kThreads = 192;                   // warp 0 loads, warp 1 MMAs, warps 2-5 compute
// TMEM columns: scores (S or S^T), dP, then the accumulators.
constexpr uint32_t kColS = 0, kColDP = 64, kColAcc0 = 128;
constexpr float kLog2e = 1.4426950408889634f;

// Sizes for a row of D elements: one or two 64-element panels (128-byte rows,
// 128-byte swizzle) at D = 64 or 128, one panel of D elements (64- or 32-byte
// rows and swizzle) at D = 32 or 16.
template <int kDim>
struct BL {
  static constexpr int kD = kDim;
  static constexpr int kPanels = kD >= 64 ? kD / 64 : 1;
  static constexpr int kPanelElems = kD >= 64 ? 64 : kD;
  static constexpr int kRowBytes = kPanelElems * 2;
  static constexpr int kTilePanel = kTile * kRowBytes;  // 128 rows of one panel
  static constexpr int kBlkPanel = kBlk * kRowBytes;
  // descriptor high word: stride between 8-row groups, sm_100 version, layout
  // type (128-byte swizzle 2, 64-byte 4, 32-byte 6)
  static constexpr uint32_t kDescHi = (uint32_t)(8 * kRowBytes >> 4) | (1u << 14) |
                                      ((kRowBytes == 128 ? 2u : kRowBytes == 64 ? 4u : 6u) << 29);
  static constexpr int kTileBytes = kPanels * kTilePanel;
  static constexpr int kBlkBytes = kPanels * kBlkPanel;
  static constexpr int kStageBytes = 2 * kBlkBytes + 1024;  // two blocks, then lse and delta (key-centric)
  static constexpr int kSmemBytes = 2 * kTileBytes + kStages * kStageBytes + 256 + 1024;
  static constexpr uint32_t kColAcc1 = kColAcc0 + kD;       // the key-centric kernel's second accumulator
  // 256 columns, two CTAs per SM at D = 64; the key-centric kernel at D = 128
  // needs 384 (512 allocated), and shared memory allows one CTA per SM there
  template <bool kKeys>
  __host__ __device__ static constexpr uint32_t tmem_cols() { return kColAcc0 + (kKeys ? 2 : 1) * kD <= 256 ? 256u : 512u; }
};

template <int kFmt>
constexpr uint32_t kIdescScore = idesc_f16kind(kTile, kBlk / 2, false, kFmt);  // 128 x 32 (a half block), B K-major
template <int kFmt, int kD>
constexpr uint32_t kIdescGrad = idesc_f16kind(kTile, kD, true, kFmt);      // 128 x D, B MN-major

struct PatGeo {
  int w, r;
  int kfull, tail;    // N div r, N mod r (TMA maps)
  FastDiv r_div;
  int n_seg;
  int tiles;          // 128-row tiles of the pattern's fullest segment
  int64_t cta_base;   // first CTA of this pattern
};

struct Params {
  Problem pb;
  BwdArgs g;
  const float* delta;  // [B, H, N] <dout_i, out_i> (key-centric kernel)
  PatGeo pat[kMaxPat];
  int64_t n_ctas;
  float scale, scale_log2;
  uint64_t wait_limit_ns;
};

// [pattern][base map / map shifted by N mod r][tile tensor 0, 1, block tensor 0, 1]
struct __align__(64) Maps {
  CUtensorMap m[kMaxPat][2][4];
};

// One sparsified segment: kept row t (t < m) at position first + r t, and
// the CTA's tile of it.
struct Unit {
  int p, b, h, first, m, tile;
};
// CTA x -> (pattern, batch, head, segment, tile).  Within a pattern the
// tiles of one segment are consecutive CTAs (they share the streamed blocks,
// which then stay in L2), longest first: the key-centric kernel's first tile
// (it meets every later query when causal) and the query-centric kernel's
// last one.
template <bool kKeys>
__device__ __forceinline__ Unit decode_cta(const Params& P, int64_t x) {
  Unit u;
  int p = 0;
  while (p + 1 < P.pb.n_pat && x >= P.pat[p + 1].cta_base) ++p;
  const PatGeo& g = P.pat[p];
  int64_t rem = x - g.cta_base;
  const int t = (int)(rem % g.tiles);
  rem /= g.tiles;
  u.tile = kKeys ? t : g.tiles - 1 - t;
  const int seg = (int)(rem % g.n_seg);
  rem /= g.n_seg;
  u.p = p;
  u.h = (int)(rem % P.pb.H);
  u.b = (int)(rem / P.pb.H);
  const int o = u.h % g.r;
  const int64_t seg_start = (int64_t)seg * g.w;
  const int64_t len = P.pb.N - seg_start < g.w ? P.pb.N - seg_start : g.w;
  u.m = len > o ? (int)((len - o + g.r - 1) / g.r) : 0;
  u.first = (int)(seg_start + o);
  return u;
}

// TMA coordinates of `need` kept rows starting at position first_pos, as in
// the forward: the base map reaches positions below r * kfull, the shifted
// map (N mod r positions further) the last ones.
struct Coord {
  int map, c, kk;
};
__device__ __forceinline__ Coord coord(const PatGeo& g, int first_pos, int need) {
  const int last_pos = first_pos + g.r * (need - 1);
  Coord t;
  t.map = last_pos >= g.r * g.kfull ? 1 : 0;
  const int x = t.map ? first_pos - g.tail : first_pos;
  t.kk = fdiv(x, g.r_div);
  t.c = x - t.kk * g.r;
  return t;
}

struct Waiter {
  volatile int* abort_flag;
  int* status;
  uint64_t limit;
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
  // every lane waits; the warp goes on only if all saw the phase
  __device__ bool wait_warp(uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, wait(bar, parity)); }
};

// dot(a, b) of two rows of kD 16-bit elements (global memory, 16-byte aligned)
template <int kFmt, int kD>
__device__ __forceinline__ float row_dot(const uint16_t* a, const uint16_t* b) {
  float d = 0.f;
#pragma unroll
  for (int c = 0; c < kD / 8; ++c) {
    const uint4 x = reinterpret_cast<const uint4*>(a)[c];
    const uint4 y = reinterpret_cast<const uint4*>(b)[c];
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w}, ys[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x0, x1, y0, y1;
      unpack2<kFmt>(xs[e], x0, x1);
      unpack2<kFmt>(ys[e], y0, y1);
      d = fmaf(x0, y0, d);
      d = fmaf(x1, y1, d);
    }
  }
  return d;
}

// P and dS of 32 streamed rows for this thread's tile row (tr), packed in
// pairs: P = 2^(s scale log2(e) - lse log2(e)), dS = P (dP - delta).
// Key-centric: the row is a key, the columns are queries (their -lse, -delta
// from shared memory, nl and nd); query-centric: the row is a query with its
// own lse2 and delta.  kMask: zero P outside the segment and, when causal,
// outside the lower triangle.
template <int kFmt, bool kKeys, bool kMask>
__device__ __forceinline__ void p_ds_half(const uint32_t (&sr)[32], const uint32_t (&dr)[32], const float* nl_col,
                                          const float* nd_col, float lse2, float delta, uint64_t sc2, int c0, int m,
                                          int tr, bool causal, uint32_t (&pk)[16], uint32_t (&dk)[16]) {
  const uint64_t nl_row = f32x2(-lse2, -lse2), nd_row = f32x2(-delta, -delta);
#pragma unroll
  for (int c = 0; c < 32; c += 4) {
    uint64_t nl[2], nd[2];
    if (kKeys) {
      const float4 l4 = *reinterpret_cast<const float4*>(nl_col + c);
      const float4 d4 = *reinterpret_cast<const float4*>(nd_col + c);
      nl[0] = f32x2(l4.x, l4.y);
      nl[1] = f32x2(l4.z, l4.w);
      nd[0] = f32x2(d4.x, d4.y);
      nd[1] = f32x2(d4.z, d4.w);
    } else {
      nl[0] = nl[1] = nl_row;
      nd[0] = nd[1] = nd_row;
    }
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      float x0, x1;
      f32x2_split(fma_f32x2(f32x2(__uint_as_float(sr[c + e]), __uint_as_float(sr[c + e + 1])), sc2, nl[e / 2]), x0,
                  x1);
      float p0 = ex2(x0), p1 = ex2(x1);
      if (kMask) {
        const int col = c0 + c + e;
        const bool v0 = col < m && (!causal || (kKeys ? col >= tr : col <= tr));
        const bool v1 = col + 1 < m && (!causal || (kKeys ? col + 1 >= tr : col + 1 <= tr));
        p0 = v0 ? p0 : 0.f;
        p1 = v1 ? p1 : 0.f;
      }
      float d0, d1;
      f32x2_split(mul_f32x2(f32x2(p0, p1),
                            add_f32x2(f32x2(__uint_as_float(dr[c + e]), __uint_as_float(dr[c + e + 1])), nd[e / 2])),
                  d0, d1);
      pk[(c + e) / 2] = pack2<kFmt>(p0, p1);
      dk[(c + e) / 2] = pack2<kFmt>(d0, d1);
    }
  }
}

// kKeys: the key-centric kernel (dk, dv); else the query-centric one (dq).
template <int kFmt, bool kKeys, int kDim>
__global__ void __launch_bounds__(kThreads, kDim <= 64 ? 2 : 1)
    bwd_tc_kernel(const __grid_constant__ Params P, const __grid_constant__ Maps maps) {
  using L = BL<kDim>;
  constexpr int kPanels = L::kPanels;
  constexpr int kTilePanel = L::kTilePanel, kBlkPanel = L::kBlkPanel;
  constexpr uint32_t kDescHi = L::kDescHi;
  constexpr int kD = L::kD, kTileBytes = L::kTileBytes, kBlkBytes = L::kBlkBytes, kStageBytes = L::kStageBytes;
  constexpr uint32_t kColAcc1 = L::kColAcc1, kTmemCols = L::template tmem_cols<kKeys>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Unit u = decode_cta<kKeys>(P, blockIdx.x);
  const int t0 = u.tile * kTile;  // first sparse row of this CTA's tile
  if (t0 >= u.m) return;                   // whole CTA, before any barrier or TMEM use
  const int nrows = u.m - t0 < kTile ? u.m - t0 : kTile;
  const bool causal = P.pb.causal != 0;
  const PatGeo& geo = P.pat[u.p];
  // streamed rows: key-centric, the queries at or after the tile (all when
  // not causal); query-centric, the keys up to the tile's last row (all)
  const int s0 = kKeys ? (causal ? t0 : 0) : 0;
  const int s1 = kKeys ? u.m : (causal ? t0 + nrows : u.m);
  const int nblk = (s1 - s0 + kBlk - 1) / kBlk;

  uint8_t* sTile0 = smem;
  uint8_t* sTile1 = smem + kTileBytes;
  uint8_t* sStage = smem + 2 * kTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + 2 * kTileBytes + kStages * kStageBytes);
  uint64_t* bar_tile = bars + 0;
  uint64_t* bar_full = bars + 1;            // [kStages]
  uint64_t* bar_empty = bars + 1 + kStages;  // [kStages]
  uint64_t* bar_s = bars + 1 + 2 * kStages;  // [2] scores of a half block in TMEM
  uint64_t* bar_p = bar_s + 2;               // [2] P and dS of a half block in TMEM
  uint64_t* bar_acc = bar_s + 4;
  uint64_t* bar_drain = bar_s + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_tile, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar_full + i, 32);  // the loading warp's 32 lanes (lane 0 with the TMA bytes)
      mbar_init(bar_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s + i, 1);
      mbar_init(bar_p + i, 128);
    }
    mbar_init(bar_acc, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < 2; ++j)
      for (int t = 0; t < 4; ++t) prefetch_tmap(&maps.m[u.p][j][t]);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  Waiter wt{abort_flag, P.pb.status, P.wait_limit_ns};
  const int64_t bhN = ((int64_t)u.b * P.pb.H + u.h) * P.pb.N;  // lse / delta row base

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    const CUtensorMap* mp0 = &maps.m[u.p][0][0];
    const CUtensorMap* mp1 = &maps.m[u.p][1][0];
    int issued = 0;
    bool ok = true;
    if (lane == 0) {
      const Coord c = coord(geo, u.first + geo.r * t0, nrows);
      const CUtensorMap* mp = c.map ? mp1 : mp0;
      mbar_arrive_expect_tx(bar_tile, 2 * kTileBytes);
#pragma unroll
      for (int pn = 0; pn < kPanels; ++pn) {
        tma_load_5d(sTile0 + pn * kTilePanel, mp + 0, bar_tile, L::kPanelElems * pn, u.h, c.c, c.kk, u.b);
        tma_load_5d(sTile1 + pn * kTilePanel, mp + 1, bar_tile, L::kPanelElems * pn, u.h, c.c, c.kk, u.b);
      }
    }
    for (int j = 0; j < nblk && ok; ++j) {
      const int st = j % kStages;
      if (j >= kStages) ok = wt.wait_warp(bar_empty + st, ((j / kStages) - 1) & 1);
      if (!ok) break;
      uint8_t* stage = sStage + st * kStageBytes;
      const int b0 = s0 + j * kBlk;
      const int need = s1 - b0 < kBlk ? s1 - b0 : kBlk;
      if (kKeys) {
        // -lse (log2 domain) and -delta of the block's queries; zero past the segment
        float* sl = reinterpret_cast<float*>(stage + 2 * kBlkBytes);
        float* sd = sl + kBlk;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int i = lane + 32 * e;
          const bool in = i < need;
          const int64_t pos = (int64_t)u.first + (int64_t)geo.r * (b0 + (in ? i : 0));
          sl[i] = in ? -P.pb.lse[bhN + pos] * kLog2e : 0.f;  // negated: the exponent's addend
          sd[i] = in ? -P.delta[bhN + pos] : 0.f;
        }
      }
      if (lane == 0) {
        const Coord c = coord(geo, u.first + geo.r * b0, need);
        const CUtensorMap* mp = c.map ? mp1 : mp0;
        mbar_arrive_expect_tx(bar_full + st, 2 * kBlkBytes);
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn) {
          tma_load_5d(stage + pn * kBlkPanel, mp + 2, bar_full + st, L::kPanelElems * pn, u.h, c.c, c.kk, u.b);
          tma_load_5d(stage + kBlkBytes + pn * kBlkPanel, mp + 3, bar_full + st, L::kPanelElems * pn, u.h, c.c,
                      c.kk, u.b);
        }
      } else {
        mbar_arrive(bar_full + st);
      }
      issued = j + 1;
    }
    // drain: every issued load has landed before the CTA may exit
    if (lane == 0) {
      if (!mbar_wait(bar_tile, 0, P.wait_limit_ns)) record_status(P.pb.status, kStatusTimeout);
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        if (!mbar_wait(bar_full + (j % kStages), (j / kStages) & 1, P.wait_limit_ns)) {
          record_status(P.pb.status, kStatusTimeout);
          break;
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t t0_lo = (smem_u32(sTile0) >> 4) | (1u << 16);
      const uint32_t t1_lo = (smem_u32(sTile1) >> 4) | (1u << 16);
      const uint32_t lbo_mn = ((uint32_t)kBlkPanel >> 4) << 16;  // the panel stride along D
      // Blocks go in two halves of 32 streamed rows, so the tensor cores work
      // on one half while the compute warps work on the other:
      //   scores(0, a) scores(0, b) | grads(j, a) scores(j+1, a) | grads(j, b) scores(j+1, b) | ...
      // A half's scores overwrite TMEM columns whose P and dS the same half's
      // gradient products (issued just before, executed in order) have read.
      auto stage_addr = [&](int j) -> uint32_t { return smem_u32(sStage + (j % kStages) * kStageBytes) >> 4; };
      auto scores = [&](int j, int hf) {
        const uint32_t b0_addr = stage_addr(j) + (uint32_t)(hf * 32 * L::kRowBytes >> 4);
        const uint32_t b1_addr = b0_addr + (kBlkBytes >> 4);
        // tile0 x block0^T and tile1 x block1^T over the half's 32 rows
        // (K-major operands, one 64-element panel of D at a time)
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn)
#pragma unroll
          for (int kk = 0; kk < L::kPanelElems / 16; ++kk)
            mma_ss(tmem + kColS + 32 * hf, desc_from(t0_lo + pn * (kTilePanel >> 4) + kk * 2, kDescHi),
                   desc_from(((b0_addr + pn * (kBlkPanel >> 4)) | (1u << 16)) + kk * 2, kDescHi), kIdescScore<kFmt>,
                   (pn > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn)
#pragma unroll
          for (int kk = 0; kk < L::kPanelElems / 16; ++kk)
            mma_ss(tmem + kColDP + 32 * hf, desc_from(t1_lo + pn * (kTilePanel >> 4) + kk * 2, kDescHi),
                   desc_from(((b1_addr + pn * (kBlkPanel >> 4)) | (1u << 16)) + kk * 2, kDescHi), kIdescScore<kFmt>,
                   (pn > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar_s + hf);
      };
      // gradients of a half: A (P or dS, packed) from TMEM, B the half's rows read MN-major
      constexpr uint32_t kStep16 = 16 * L::kRowBytes >> 4;  // 16 rows of an MN-major operand
      auto grads = [&](int j, int hf) {
        const uint32_t b0_addr = stage_addr(j) + (uint32_t)(hf * 32 * L::kRowBytes >> 4);
        const uint32_t b1_addr = b0_addr + (kBlkBytes >> 4);
#pragma unroll
        for (int kk = 0; kk < kBlk / 32; ++kk) {
          const uint32_t acc = (j > 0 || hf > 0 || kk > 0) ? 1u : 0u;
          if (kKeys) {
            // dV += P^T dout (block 1), dK += dS^T Q (block 0)
            mma_ts(tmem + kColAcc0, tmem + kColS + 32 * hf + kk * 8, desc_from((b1_addr | lbo_mn) + kk * kStep16, kDescHi),
                   kIdescGrad<kFmt, kD>, acc);
            mma_ts(tmem + kColAcc1, tmem + kColDP + 32 * hf + kk * 8, desc_from((b0_addr | lbo_mn) + kk * kStep16, kDescHi),
                   kIdescGrad<kFmt, kD>, acc);
          } else {
            // dQ += dS K (block 0)
            mma_ts(tmem + kColAcc0, tmem + kColDP + 32 * hf + kk * 8, desc_from((b0_addr | lbo_mn) + kk * kStep16, kDescHi),
                   kIdescGrad<kFmt, kD>, acc);
          }
        }
      };
      bool ok = wt.wait(bar_tile, 0) && wt.wait(bar_full + 0, 0);
      if (ok) {
        tc_fence_after();
        scores(0, 0);
        scores(0, 1);
      }
      for (int j = 0; j < nblk && ok; ++j) {
        const bool more = j + 1 < nblk;
        ok = wt.wait(bar_p + 0, j & 1);
        if (!ok) break;
        tc_fence_after();
        grads(j, 0);
        if (more) {
          ok = wt.wait(bar_full + (j + 1) % kStages, ((j + 1) / kStages) & 1);
          if (!ok) break;
          tc_fence_after();
          scores(j + 1, 0);
        }
        ok = wt.wait(bar_p + 1, j & 1);
        if (!ok) break;
        tc_fence_after();
        grads(j, 1);
        tc_commit(bar_empty + j % kStages);  // the block's shared memory is free once its products ran
        if (more) scores(j + 1, 1);
      }
      if (ok) tc_commit(bar_acc);
      // drain: all issued MMAs complete before TMEM is released
      tc_commit(bar_drain);
      if (!mbar_wait(bar_drain, 0, P.wait_limit_ns)) record_status(P.pb.status, kStatusTimeout);
    }
  } else {
    // ------------------------------------------------------------ P, dS and the epilogue
    const int row = 32 * (warp & 3) + lane;  // TMEM lane = tile row
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int tr = t0 + row;                  // sparse index of this thread's row
    const bool row_ok = row < nrows;
    const int64_t pos = (int64_t)u.first + (int64_t)geo.r * (row_ok ? tr : t0);
    const int64_t elem = (((int64_t)u.b * P.pb.N + pos) * P.pb.H + u.h) * kD;
    float lse2 = 0.f, delta = 0.f;
    if (!kKeys && row_ok) {
      lse2 = P.pb.lse[bhN + pos] * kLog2e;
      delta = row_dot<kFmt, kD>(static_cast<const uint16_t*>(P.g.dout) + elem,
                            static_cast<const uint16_t*>(P.g.out) + elem);
    }
    const uint64_t sc2 = f32x2(P.scale_log2, P.scale_log2);
    bool ok = true;
    for (int j = 0; j < nblk && ok; ++j) {
      const int st = j % kStages;
      const float* sl = reinterpret_cast<const float*>(sStage + st * kStageBytes + 2 * kBlkBytes);
      const float* sd = sl + kBlk;
      if (kKeys) ok = wt.wait_warp(bar_full + st, (j / kStages) & 1);
      if (!ok) break;
      const int b0 = s0 + j * kBlk;
      // every (row, column) pair of the block real: no masking needed
      const bool full = b0 + kBlk <= u.m && (!causal || (kKeys ? b0 >= tr : b0 + kBlk - 1 <= tr));
      // two halves of 32 streamed rows, each as soon as its scores are in
      // TMEM: scores and dP in, P and dS (packed pairs) out over the first 16
      // columns of the half's own 32
#pragma unroll 1
      for (int hf = 0; hf < 2 && ok; ++hf) {
        ok = wt.wait_warp(bar_s + hf, j & 1);
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[32], dr[32];
        LN_TMEM_LD32(tmem + lane_base + kColS + 32 * hf, sr);
        LN_TMEM_LD32(tmem + lane_base + kColDP + 32 * hf, dr);
        tmem_wait_ld();
        uint32_t pk[16], dk[16];
        const int c0 = b0 + 32 * hf;  // sparse index of the half's first streamed row
        if (full)
          p_ds_half<kFmt, kKeys, false>(sr, dr, sl + 32 * hf, sd + 32 * hf, lse2, delta, sc2, c0, u.m, tr, causal, pk, dk);
        else
          p_ds_half<kFmt, kKeys, true>(sr, dr, sl + 32 * hf, sd + 32 * hf, lse2, delta, sc2, c0, u.m, tr, causal, pk, dk);
        if (kKeys) LN_TMEM_ST16(tmem + lane_base + kColS + 32 * hf, pk);
        LN_TMEM_ST16(tmem + lane_base + kColDP + 32 * hf, dk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p + hf);
      }
    }
    if (ok) ok = wt.wait_warp(bar_acc, 0);
    if (ok) {
      tc_fence_after();
      // key-centric: dV (no scale) then dK (times 1/sqrt(D)); query-centric: dQ
#pragma unroll 1
      for (int a = 0; a < (kKeys ? 2 : 1); ++a) {
        float* dst = kKeys ? (a == 0 ? P.g.dv : P.g.dk) : P.g.dq;
        const float sc = (kKeys && a == 0) ? 1.f : P.scale;
        constexpr int kChunk = kD < 32 ? kD : 32;  // accumulator columns per TMEM load
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += kChunk) {
          uint32_t acc[kChunk];
          if constexpr (kChunk == 32) {
            LN_TMEM_LD32(tmem + lane_base + (a == 0 ? kColAcc0 : kColAcc1) + c0, acc);
          } else {
            LN_TMEM_LD16(tmem + lane_base + (a == 0 ? kColAcc0 : kColAcc1) + c0, acc);
          }
          tmem_wait_ld();
          if (row_ok) {
            float4* d4 = reinterpret_cast<float4*>(dst + elem + c0);
#pragma unroll
            for (int c = 0; c < kChunk / 4; ++c)
              atomicAdd(d4 + c, make_float4(__uint_as_float(acc[4 * c]) * sc, __uint_as_float(acc[4 * c + 1]) * sc,
                                            __uint_as_float(acc[4 * c + 2]) * sc,
                                            __uint_as_float(acc[4 * c + 3]) * sc));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// delta_i = <dout_i, out_i> for every row, into [B, H, N]; one thread per row.
template <int kFmt, int kD>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const Problem pb, const uint16_t* out, const uint16_t* dout,
                                                        float* delta) {
  const int64_t rows = pb.B * pb.N * pb.H;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t h = i % pb.H, n = (i / pb.H) % pb.N, b = i / (pb.H * pb.N);
    delta[(b * pb.H + h) * pb.N + n] = row_dot<kFmt, kD>(dout + i * kD, out + i * kD);
  }
}

// View [B, N, H, D] (16-bit elements, starting `shift` positions in) as
// (d, h, c, k, b), position = r k + c; boxes of one 64-element panel of D by
// box_rows consecutive k.
bool encode(EncodeTiledFn enc, CUtensorMap* map, const void* base, const Problem& p, int64_t r, int64_t shift,
            int64_t kcount, int box_rows) {
  const int64_t es = 2, D = p.D;
  const char* ptr = static_cast<const char*>(base) + shift * p.H * D * es;
  cuuint64_t dims[5] = {(cuuint64_t)D, (cuuint64_t)p.H, (cuuint64_t)r, (cuuint64_t)kcount, (cuuint64_t)p.B};
  cuuint64_t strides[4] = {(cuuint64_t)(D * es), (cuuint64_t)(p.H * D * es), (cuuint64_t)(r * p.H * D * es),
                           (cuuint64_t)(p.N * p.H * D * es)};
  const int64_t pe = D >= 64 ? 64 : D;  // elements of a panel row
  cuuint32_t box[5] = {(cuuint32_t)pe, 1, 1, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  const CUtensorMapDataType ty =
      p.dtype == LONGNET_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  return enc(map, ty, 5, const_cast<char*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             pe == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : pe == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// CTAs and the per-pattern geometry; false when the shape is outside this
// family.
bool geometry(const Problem& p, Params* P) {
  if ((p.dtype != LONGNET_DTYPE_BF16 && p.dtype != LONGNET_DTYPE_F16) ||
      (p.D != 16 && p.D != 32 && p.D != 64 && p.D != 128) || p.qk_norm)
    return false;
  if (p.n_pat > kMaxPat || p.N > ((int64_t)1 << 30) || p.H > 65535 || p.B > 65535) return false;
  int64_t ctas = 0;
  for (int i = 0; i < p.n_pat; ++i) {
    const int64_t w = p.w[i] < p.N ? p.w[i] : p.N, r = p.r[i];
    if (r > 4096) return false;
    const int64_t tail = p.N % r;
    // a 128-row box never needs both the first and the last N mod r positions
    if (tail > 0 && p.N < kTile * r + 2 * tail) return false;
    if (p.N / r < 1) return false;
    const int64_t n_seg = (p.N + w - 1) / w;
    const int64_t tiles = ((w + r - 1) / r + kTile - 1) / kTile;
    if (P) {
      PatGeo& g = P->pat[i];
      g.w = (int)w;
      g.r = (int)r;
      g.kfull = (int)(p.N / r);
      g.tail = (int)tail;
      g.r_div = make_fastdiv(r);
      g.n_seg = (int)n_seg;
      g.tiles = (int)tiles;
      g.cta_base = ctas;
    }
    ctas += p.B * p.H * n_seg * tiles;
    if (ctas > 0x7fffffffLL) return false;
  }
  if (P) P->n_ctas = ctas;
  return ctas > 0;
}

}  // namespace tb

bool tcgen05_backward_supports(const Problem& p) {
  return tb::geometry(p, nullptr);
}

int launch_tcgen05_backward(const Problem& p, const BwdArgs& g, cudaStream_t stream) {
  using namespace tb;
  static Params P;  // host staging in static storage (the library allocates nothing)
  static Maps mk, mq;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  memset(&P, 0, sizeof(P));
  if (!geometry(p, &P)) return LONGNET_ERR_UNSUPPORTED;
  EncodeTiledFn enc = get_encoder();
  if (!enc) return LONGNET_ERR_CUDA;
  P.pb = p;
  P.g = g;
  P.delta = g.dq;  // delta lives in the dq buffer until the dq kernel
  P.scale = 1.f / sqrtf((float)p.D);
  P.scale_log2 = kLog2e * P.scale;
  P.wait_limit_ns = kWaitLimitNs;
  // key-centric maps: K, V tiles (128 rows), Q, dout blocks (64 rows);
  // query-centric: Q, dout tiles, K, V blocks
  const void* kc[4] = {p.k, p.v, p.q, g.dout};
  const void* qc[4] = {p.q, g.dout, p.k, p.v};
  for (int i = 0; i < p.n_pat; ++i) {
    const PatGeo& pg = P.pat[i];
    for (int t = 0; t < 4; ++t) {
      const int rows = t < 2 ? kTile : kBlk;
      for (int sh = 0; sh < 2; ++sh) {
        const int64_t shift = sh ? pg.tail : 0;
        if (!encode(enc, &mk.m[i][sh][t], kc[t], p, pg.r, shift, pg.kfull, rows) ||
            !encode(enc, &mq.m[i][sh][t], qc[t], p, pg.r, shift, pg.kfull, rows))
          return LONGNET_ERR_CUDA;
      }
    }
  }
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  const bool f16 = p.dtype == LONGNET_DTYPE_F16;
  using KFn = void (*)(Params, Maps);
  using DFn = void (*)(const Problem, const uint16_t*, const uint16_t*, float*);
  const int di = p.D == 16 ? 0 : p.D == 32 ? 1 : p.D == 64 ? 2 : 3;
  static const KFn kk_tab[2][4] = {
      {bwd_tc_kernel<kFmtBF16, true, 16>, bwd_tc_kernel<kFmtBF16, true, 32>, bwd_tc_kernel<kFmtBF16, true, 64>,
       bwd_tc_kernel<kFmtBF16, true, 128>},
      {bwd_tc_kernel<kFmtF16, true, 16>, bwd_tc_kernel<kFmtF16, true, 32>, bwd_tc_kernel<kFmtF16, true, 64>,
       bwd_tc_kernel<kFmtF16, true, 128>}};
  static const KFn kq_tab[2][4] = {
      {bwd_tc_kernel<kFmtBF16, false, 16>, bwd_tc_kernel<kFmtBF16, false, 32>, bwd_tc_kernel<kFmtBF16, false, 64>,
       bwd_tc_kernel<kFmtBF16, false, 128>},
      {bwd_tc_kernel<kFmtF16, false, 16>, bwd_tc_kernel<kFmtF16, false, 32>, bwd_tc_kernel<kFmtF16, false, 64>,
       bwd_tc_kernel<kFmtF16, false, 128>}};
  static const DFn kd_tab[2][4] = {
      {bwd_delta_kernel<kFmtBF16, 16>, bwd_delta_kernel<kFmtBF16, 32>, bwd_delta_kernel<kFmtBF16, 64>,
       bwd_delta_kernel<kFmtBF16, 128>},
      {bwd_delta_kernel<kFmtF16, 16>, bwd_delta_kernel<kFmtF16, 32>, bwd_delta_kernel<kFmtF16, 64>,
       bwd_delta_kernel<kFmtF16, 128>}};
  static const int smem_tab[4] = {BL<16>::kSmemBytes, BL<32>::kSmemBytes, BL<64>::kSmemBytes, BL<128>::kSmemBytes};
  const KFn kern_k = kk_tab[f16][di], kern_q = kq_tab[f16][di];
  const DFn kern_d = kd_tab[f16][di];
  const int kSmemBytes = smem_tab[di];
  static bool attr_set[64][2][4] = {};
  if (!attr_set[dev][f16][di]) {
    if (cudaFuncSetAttribute(kern_k, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(kern_q, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess) {
      cudaGetLastError();
      return LONGNET_ERR_CUDA;
    }
    attr_set[dev][f16][di] = true;
  }
  int n_sm = 148;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t rows = p.B * p.N * p.H;
  int64_t dblocks = (rows + 255) / 256;
  if (dblocks > (int64_t)n_sm * 16) dblocks = (int64_t)n_sm * 16;
  const size_t bytes = sizeof(float) * (size_t)(rows * p.D);
  // delta into the dq buffer; dk, dv zeroed; keys; dq zeroed; queries
  kern_d<<<(unsigned)dblocks, 256, 0, stream>>>(p, static_cast<const uint16_t*>(g.out),
                                                static_cast<const uint16_t*>(g.dout), g.dq);
  if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  if (cudaMemsetAsync(g.dk, 0, bytes, stream) != cudaSuccess || cudaMemsetAsync(g.dv, 0, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  const dim3 grid((unsigned)P.n_ctas);
  kern_k<<<grid, kThreads, kSmemBytes, stream>>>(P, mk);
  if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  if (cudaMemsetAsync(g.dq, 0, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  kern_q<<<grid, kThreads, kSmemBytes, stream>>>(P, mq);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

}  // namespace longnet
