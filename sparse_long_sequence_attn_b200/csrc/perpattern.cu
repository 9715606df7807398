// Kernel family PATTERNS: the multi-pattern dilated-attention forward one
// pattern at a time, on the 5th-generation tensor cores, for bf16 or fp16 at
// D = 16, 32, 64 or 128 and any number of patterns.
//
// What it computes is the forward of the fused tcgen05 family ("LONGNET:
// Scaling Transformer to 1 billion tokens", section "LongNet's attention
// allocation principle"; "LongNet论文精读", section "Dilated Attention的工作原理"):
// per pattern (w, r), segments of w tokens, head h keeping the rows o + r k
// (o = h mod r), softmax(Q K^T / sqrt(D)) V on each sparsified segment, and the
// patterns combined per row with weights equal to their softmax denominators
// ("LONGNET: Scaling Transformer to 1 billion tokens", section "Token
// expansion reaches 1 billion+").  The combination is done through HBM
// instead of shared memory: out and lse first hold 0 and -inf (a row no
// pattern keeps stays so), then each pattern's launch merges its rows into
// them, out = (e^lse out + e^lse_p O_p) / (e^lse + e^lse_p), lse = logaddexp.
// That frees the shared memory the fused kernel spends on parking slots, so
// wider heads (D = 128: 256-byte rows) and more patterns fit.
//
// Design (one launch per pattern):
//  * One CTA per (batch, head, segment, 128-row tile of the sparsified
//    segment), tiles of a segment consecutive (they stream the same key
//    blocks, which then stay in L2), the longest first.
//  * Warp 0 loads through the dilated 5-D TMA maps (position = r k + c):
//    the Q tile once, then 64-key K and V blocks through a ring; a row of
//    D = 128 is two 128-byte swizzle panels.  Warp 1 issues S = Q K^T into
//    one of two TMEM score buffers and, one block behind, O += P V with P
//    read from TMEM.  Warps 2-5, one thread per row: online softmax in fp32
//    (exp2 of scaled scores, O rescaled in TMEM only when the row maximum grows
//    by more than 2^8), P written back over its score buffer in the input
//    format, and at the end the merge into out and lse.
//  * TMEM: two 64-column score buffers and a D-column O: 256 columns, two
//    CTAs per SM.
//  * The pattern launches overlap: each is a programmatic dependent launch,
//    whose CTAs compute their attention while the previous launch finishes
//    and wait for it (griddepcontrol.wait) only before the merge, so a
//    launch's last, longest CTAs do not leave the GPU idle.
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
namespace pp {
using namespace tc;

constexpr int kTile = 128;   // rows per CTA (M of the MMAs)
constexpr int kBlk = 64;     // keys per block (N of S = Q K^T)
constexpr int kThreads = 192;      // loads, MMA issue, four softmax warps
constexpr int kThreadsNorm = 256;  // with qk_norm, and two warps for the key norms
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColO = 128;  // scores at 0 and 64
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.69314718055994531f;

// Rows of D elements as swizzle panels: D = 64 or 128 is one or two panels of
// 64 elements (128-byte rows, 128-byte swizzle); D = 32 or 16 is one panel of
// D elements (64- or 32-byte rows, 64- or 32-byte swizzle).  Ring stages: 3 up
// to D = 64, 2 at D = 128 (two CTAs per SM).
template <int kD>
struct Layout {
  static constexpr int kPanels = kD >= 64 ? kD / 64 : 1;
  static constexpr int kPanelElems = kD >= 64 ? 64 : kD;
  static constexpr int kRowBytes = kPanelElems * 2;  // one panel row
  static constexpr int kQPanel = kTile * kRowBytes;
  static constexpr int kKVPanel = kBlk * kRowBytes;
  // descriptor high word: stride between 8-row groups, sm_100 version, layout
  // type (128-byte swizzle 2, 64-byte 4, 32-byte 6)
  static constexpr uint32_t kDescHi = (uint32_t)(8 * kRowBytes >> 4) | (1u << 14) |
                                      ((kRowBytes == 128 ? 2u : kRowBytes == 64 ? 4u : 6u) << 29);
  static constexpr int kStages = kD <= 64 ? 3 : 2;
  static constexpr int kQBytes = kPanels * kQPanel;
  static constexpr int kStageBytes = 2 * kPanels * kKVPanel;  // K panels, then V panels
  static constexpr int kBars = kQBytes + kStages * kStageBytes;
  // at least 80 KB, so no third CTA (whose 256 TMEM columns would not fit)
  // shares an SM
  // barriers (256 B), then qk_norm's inverse key norms [2][kBlk] (512 B)
  static constexpr int kSmem = kBars + 768 + 1024 > 80 * 1024 ? kBars + 768 + 1024 : 80 * 1024;
};

struct Params {
  Problem pb;
  int p;              // the pattern of this launch
  int w, r;           // its segment length (at most N) and dilation
  int kfull, tail;    // N div r, N mod r (TMA maps)
  FastDiv r_div;
  int n_seg, tiles;   // segments, 128-row tiles of the fullest one
  int first_call;     // no earlier pattern has written out and lse
  float scale_log2;
  uint64_t wait_limit_ns;
};

struct __align__(64) Maps {
  CUtensorMap m[2][3];  // [base / shifted by N mod r][q, k, v]
};

struct Coord {
  int map, c, kk;
};
__device__ __forceinline__ Coord coord(const Params& P, int first_pos, int need) {
  const int last_pos = first_pos + P.r * (need - 1);
  Coord t;
  t.map = last_pos >= P.r * P.kfull ? 1 : 0;
  const int x = t.map ? first_pos - P.tail : first_pos;
  t.kk = fdiv(x, P.r_div);
  t.c = x - t.kk * P.r;
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
  __device__ bool wait_warp(uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, wait(bar, parity)); }
};

// kNorm: LONGNET_FLAG_QK_NORM, q and k rows taken at unit L2 norm: the
// scores are scaled in fp32 by the row's and the key's inverse norms, which
// bounds a scaled logit by the softmax scale (a cosine times it), the fixed
// stabiliser of every block.
template <int kFmt, int kD, bool kNorm>
__global__ void __launch_bounds__(kNorm ? kThreadsNorm : kThreads, 2)
    pp_fwd_kernel(const __grid_constant__ Params P, const __grid_constant__ Maps maps) {
  using L = Layout<kD>;
  constexpr int kPanels = L::kPanels;
  constexpr int kQPanel = L::kQPanel, kKVPanel = L::kKVPanel;
  constexpr uint32_t kDescHi = L::kDescHi;
  // O moves between TMEM and registers kOChunk columns at a time (16 at D = 16)
  constexpr int kOChunk = kD < 32 ? kD : 32;
  auto o_load = [](uint32_t taddr, uint32_t(&r)[kOChunk]) {
    if constexpr (kOChunk == 32) {
      LN_TMEM_LD32(taddr, r);
    } else {
      LN_TMEM_LD16(taddr, r);
    }
    tmem_wait_ld();
  };
  auto o_store = [](uint32_t taddr, uint32_t(&r)[kOChunk]) {
    if constexpr (kOChunk == 32) {
      LN_TMEM_ST32(taddr, r);
    } else {
      LN_TMEM_ST16(taddr, r);
    }
  };
  constexpr int S = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // the next pattern's launch may start as soon as every CTA of this one has:
  // its attention reads only q, k and v, and its merge waits for this grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // CTA -> (batch, head of the part, segment, tile): tiles fastest, longest first
  int64_t rem = blockIdx.x;
  const int tile = P.tiles - 1 - (int)(rem % P.tiles);
  rem /= P.tiles;
  const int seg = (int)(rem % P.n_seg);
  rem /= P.n_seg;
  const int Hr = (int)(P.pb.h1 - P.pb.h0);
  const int h = (int)P.pb.h0 + (int)(rem % Hr);
  const int b = (int)(rem / Hr);
  const int o = h % P.r;
  const int64_t seg_start = (int64_t)seg * P.w;
  const int64_t len = P.pb.N - seg_start < P.w ? P.pb.N - seg_start : P.w;
  const int m = len > o ? (int)((len - o + P.r - 1) / P.r) : 0;
  const int first = (int)(seg_start + o);
  const int t0 = tile * kTile;
  if (t0 >= m) return;  // whole CTA, before any barrier or TMEM use
  const int nrows = m - t0 < kTile ? m - t0 : kTile;
  // rows of the tile inside the computed part [q0, q1)?
  {
    const int64_t lo = first + (int64_t)P.r * t0, hi = first + (int64_t)P.r * (t0 + nrows - 1);
    if (hi < P.pb.q0 || lo >= P.pb.q1) return;
  }
  const bool causal = P.pb.causal != 0;
  const int s1 = causal ? t0 + nrows : m;  // keys [0, s1) of the segment
  const int nblk = (s1 + kBlk - 1) / kBlk;

  uint8_t* sQ = smem;
  uint8_t* sStage = smem + L::kQBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBars);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_full = bars + 1;       // [S]
  uint64_t* bar_empty = bars + 1 + S;  // [S]
  uint64_t* bar_s = bars + 1 + 2 * S;  // [2] score buffers
  uint64_t* bar_p = bar_s + 2;         // [2]
  uint64_t* bar_od = bar_s + 4;        // O += P V of a block done
  uint64_t* bar_of = bar_s + 5;        // the last one done
  uint64_t* bar_drain = bar_s + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_s + 7);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* bar_ikn = bar_s + 8;  // qk_norm: [2] block parity, one arrival per lane of the norm warps
  float* ikn = reinterpret_cast<float*>(smem + L::kBars + 256);  // qk_norm: [2][kBlk]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < S; ++i) {
      mbar_init(bar_full + i, 1);
      mbar_init(bar_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_s + i, 1);
      mbar_init(bar_p + i, 128);
    }
    mbar_init(bar_od, 1);
    mbar_init(bar_of, 1);
    mbar_init(bar_drain, 1);
    mbar_init(bar_ikn + 0, 64);
    mbar_init(bar_ikn + 1, 64);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int j = 0; j < 2; ++j)
      for (int t = 0; t < 3; ++t) prefetch_tmap(&maps.m[j][t]);
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
  // qk_norm: sum of squares of a row of 16-bit elements in a swizzled tile;
  // the swizzle only permutes the 16-byte chunks inside each row's bytes, so
  // the row's chunks (panel after panel) are summed in place
  auto row_sumsq = [](const uint8_t* tile, int panel_bytes, int r) -> float {
    constexpr int kCpr = L::kRowBytes / 16;  // chunks per panel row
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < kD / 8; ++i) {
      const uint4 u =
          *reinterpret_cast<const uint4*>(tile + (i / kCpr) * panel_bytes + r * L::kRowBytes + (i % kCpr) * 16);
      const uint32_t wv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float lo, hi;
        unpack2<kFmt>(wv[e], lo, hi);
        acc = fmaf(lo, lo, fmaf(hi, hi, acc));
      }
    }
    return acc;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ loads
    if (lane == 0) {
      bool ok = true;
      {
        const Coord c = coord(P, first + P.r * t0, nrows);
        mbar_arrive_expect_tx(bar_q, L::kQBytes);
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn)
          tma_load_5d(sQ + pn * kQPanel, &maps.m[c.map][0], bar_q, L::kPanelElems * pn, h, c.c, c.kk, b);
      }
      int issued = 0;
      for (int j = 0; j < nblk && ok; ++j) {
        const int st = j % S;
        if (j >= S) ok = wt.wait(bar_empty + st, ((j / S) - 1) & 1);
        if (!ok) break;
        const int b0 = j * kBlk;
        const int need = s1 - b0 < kBlk ? s1 - b0 : kBlk;
        const Coord c = coord(P, first + P.r * b0, need);
        uint8_t* stage = sStage + st * L::kStageBytes;
        mbar_arrive_expect_tx(bar_full + st, L::kStageBytes);
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn) {
          tma_load_5d(stage + pn * kKVPanel, &maps.m[c.map][1], bar_full + st, L::kPanelElems * pn, h, c.c, c.kk,
                      b);
          tma_load_5d(stage + (kPanels + pn) * kKVPanel, &maps.m[c.map][2], bar_full + st, L::kPanelElems * pn, h,
                      c.c, c.kk, b);
        }
        issued = j + 1;
      }
      // drain: every issued load has landed before the CTA may exit
      if (!mbar_wait(bar_q, 0, P.wait_limit_ns)) record_status(P.pb.status, kStatusTimeout);
      for (int j = issued > S ? issued - S : 0; j < issued; ++j)
        if (!mbar_wait(bar_full + (j % S), (j / S) & 1, P.wait_limit_ns)) {
          record_status(P.pb.status, kStatusTimeout);
          break;
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_f16kind(kTile, kBlk, false, kFmt);  // 128 x 64, B K-major
      constexpr uint32_t kIdO = idesc_f16kind(kTile, kD, true, kFmt);     // 128 x D, B MN-major
      const uint32_t q_lo = smem_u32(sQ) >> 4;
      const uint32_t lbo_mn = ((uint32_t)kKVPanel >> 4) << 16;  // V's panel stride along N
      auto pv = [&](int jj) -> bool {
        if (!wt.wait(bar_p + (jj & 1), (jj >> 1) & 1)) return false;
        tc_fence_after();
        const uint32_t v_lo = (smem_u32(sStage + (jj % S) * L::kStageBytes) >> 4) + (uint32_t)(kPanels * kKVPanel >> 4);
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk)
          mma_ts(tmem + kColO, tmem + 64 * (jj & 1) + kk * 8,
                 desc_from((v_lo | lbo_mn) + kk * (16 * L::kRowBytes >> 4), kDescHi), kIdO,
                 (jj > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar_empty + jj % S);
        tc_commit(bar_od);
        return true;
      };
      bool ok = wt.wait(bar_q, 0);
      for (int j = 0; j < nblk && ok; ++j) {
        const int st = j % S;
        ok = wt.wait(bar_full + st, (j / S) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint32_t k_lo = smem_u32(sStage + st * L::kStageBytes) >> 4;
        // S(j) = Q K^T over D (a 64-element panel at a time)
#pragma unroll
        for (int pn = 0; pn < kPanels; ++pn)
#pragma unroll
          for (int kk = 0; kk < L::kPanelElems / 16; ++kk)
            mma_ss(tmem + 64 * (j & 1), desc_from(((q_lo + pn * (kQPanel >> 4)) | (1u << 16)) + kk * 2, kDescHi),
                   desc_from(((k_lo + pn * (kKVPanel >> 4)) | (1u << 16)) + kk * 2, kDescHi), kIdS,
                   (pn > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar_s + (j & 1));
        if (j > 0) ok = pv(j - 1);
      }
      if (ok) ok = pv(nblk - 1);
      if (ok) tc_commit(bar_of);
      tc_commit(bar_drain);
      if (!mbar_wait(bar_drain, 0, P.wait_limit_ns)) record_status(P.pb.status, kStatusTimeout);
    }
  } else if (kNorm && warp >= 6) {
    // ------------------------------------------------------------ key norms (qk_norm)
    // Per block: the inverse norms of its 64 K rows (the K block stays in its
    // stage until its P V has run) into the array of the block's parity, once
    // the block has landed and, from block 2 on, every softmax thread has
    // written block j - 2's P, which it does after its last read of that
    // block's array (the same parity).  Warps 6 and 7, one key per lane.
    bool ok = true;
    for (int j = 0; j < nblk && ok; ++j) {
      ok = wt.wait_warp(bar_full + j % S, (j / S) & 1);
      if (ok && j >= 2) ok = wt.wait_warp(bar_p + (j & 1), ((j - 2) >> 1) & 1);
      if (!ok) break;
      const uint8_t* kb = sStage + (j % S) * L::kStageBytes;
      const int kr = 32 * (warp - 6) + lane;
      ikn[(j & 1) * kBlk + kr] = 1.f / fmaxf(sqrtf(row_sumsq(kb, kKVPanel, kr)), 1e-12f);
      mbar_arrive(bar_ikn + (j & 1));
    }
  } else {
    // ------------------------------------------------------------ softmax and the merge
    const int row = 32 * (warp & 3) + lane;  // TMEM lane = tile row
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const int tr = t0 + row;
    float m_use = -INFINITY, l_run = 0.f;
    bool ok = true;
    float row_scale = P.scale_log2;  // with qk_norm times the row's inverse q norm
    if constexpr (kNorm) {
      ok = wt.wait_warp(bar_q, 0);
      if (ok) row_scale = P.scale_log2 / fmaxf(sqrtf(row_sumsq(sQ, kQPanel, row)), 1e-12f);
    }
    const uint64_t sc2 = f32x2(row_scale, row_scale);
    for (int j = 0; j < nblk && ok; ++j) {
      if constexpr (kNorm) {
        // this block's inverse key norms, from the norm warp
        ok = wt.wait_warp(bar_ikn + (j & 1), (j >> 1) & 1);
        if (!ok) break;
      }
      ok = wt.wait_warp(bar_s + (j & 1), (j >> 1) & 1);
      if (!ok) break;
      tc_fence_after();
      const uint32_t s_col = tmem + lane_base + 64 * (j & 1);
      uint32_t sr[kBlk];
      LN_TMEM_LD32(s_col, (sr + 0));
      LN_TMEM_LD32(s_col + 32, (sr + 32));
      tmem_wait_ld();
      // keys past the segment, and after the row when causal
      const int b0 = j * kBlk;
      const int lim = (causal ? (tr < m ? tr : m - 1) : m - 1) - b0;  // last valid column
      if (lim < kBlk - 1) {
#pragma unroll
        for (int c = 0; c < kBlk; ++c)
          if (c > lim) sr[c] = __float_as_uint(-INFINITY);
      }
      float corr = 1.f;
      bool rescale = false;
      if constexpr (kNorm) {
        m_use = P.scale_log2;  // the bound of every scaled logit
      } else {
        float pm[8];
#pragma unroll
        for (int q8 = 0; q8 < 8; ++q8) pm[q8] = __uint_as_float(sr[q8]);
#pragma unroll
        for (int c = 8; c < kBlk; ++c) pm[c & 7] = fmaxf(pm[c & 7], __uint_as_float(sr[c]));
        const float mx = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])), fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        const float m_blk = mx * P.scale_log2;
        if (m_blk > m_use + 8.f || m_use == -INFINITY) {
          if (m_blk != -INFINITY) {
            if (m_use != -INFINITY) {
              corr = ex2(m_use - m_blk);
              rescale = true;
            }
            m_use = m_blk;
          }
        }
      }
      // P = 2^(s scale - m) in the input format over the first 32 columns
      float ps[8];
      {
        uint32_t pk[32];
        const uint64_t nm2 = f32x2(-m_use, -m_use);
        uint64_t ls[4] = {0, 0, 0, 0};
        const ulonglong2* ik2 = reinterpret_cast<const ulonglong2*>(ikn + (j & 1) * kBlk);  // qk_norm
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          uint64_t coef = sc2;  // the scale of keys 2c and 2c + 1
          if constexpr (kNorm) {
            const ulonglong2 pr = ik2[c >> 1];
            coef = mul_f32x2((c & 1) ? pr.y : pr.x, sc2);
          }
          float xa, xb;
          f32x2_split(fma_f32x2(f32x2(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), coef, nm2), xa, xb);
          const float a = ex2(xa), bq = ex2(xb);
          ls[c & 3] = add_f32x2(ls[c & 3], f32x2(a, bq));
          pk[c] = pack2<kFmt>(a, bq);
        }
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) f32x2_split(ls[q4], ps[2 * q4], ps[2 * q4 + 1]);
        LN_TMEM_ST32(s_col, pk);
      }
      tmem_wait_st();
      l_run = l_run * corr + (((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7])));
      if (j > 0 && __any_sync(0xffffffffu, rescale)) {
        // O of blocks before j - 1 is final (their products ran before S(j));
        // the one of block j - 1 is the latest O += P V pending
        ok = wt.wait_warp(bar_od, (j - 1) & 1);
        if (!ok) break;
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < kD; c0 += kOChunk) {
          uint32_t rr[kOChunk];
          o_load(tmem + lane_base + kColO + c0, rr);
#pragma unroll
          for (int c = 0; c < kOChunk; ++c) rr[c] = __float_as_uint(__uint_as_float(rr[c]) * corr);
          o_store(tmem + lane_base + kColO + c0, rr);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(bar_p + (j & 1));
    }
    if (ok) ok = wt.wait_warp(bar_of, 0);
    // out and lse as the previous launch (the init pass or the previous
    // pattern) left them: that grid has completed and its writes are visible
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (ok) {
      tc_fence_after();
      const int64_t pos = (int64_t)first + (int64_t)P.r * (tr < m ? tr : t0);
      const bool write = row < nrows && pos >= P.pb.q0 && pos < P.pb.q1;
      const int64_t elem = (((int64_t)b * P.pb.N + pos) * P.pb.H + h) * kD;
      const int64_t lidx = ((int64_t)b * P.pb.H + h) * P.pb.N + pos;
      // this pattern's lse (log2 domain) and the weights of the merge
      const float lse_p = m_use + __log2f(l_run);
      float old2 = -INFINITY;
      if (write && !P.first_call && P.pb.lse) old2 = P.pb.lse[lidx] * kLog2e;
      const float mx = fmaxf(old2, lse_p);
      const float wa = ex2(old2 - mx), wb = ex2(lse_p - mx);
      const float inv = 1.f / (wa + wb);
      const float ca = wa * inv, cb = wb * inv / l_run;
      uint16_t* orow = static_cast<uint16_t*>(P.pb.out) + elem;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += kOChunk) {
        uint32_t rr[kOChunk];
        o_load(tmem + lane_base + kColO + c0, rr);
        if (write) {
#pragma unroll
          for (int q = 0; q < kOChunk / 8; ++q) {  // 8 elements (16 bytes) at a time
            uint4 old = make_uint4(0, 0, 0, 0);
            if (!P.first_call) old = reinterpret_cast<const uint4*>(orow + c0)[q];
            const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
            uint32_t nw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float a0, a1;
              unpack2<kFmt>(ow[e], a0, a1);
              const float n0 = fmaf(__uint_as_float(rr[8 * q + 2 * e]), cb, a0 * ca);
              const float n1 = fmaf(__uint_as_float(rr[8 * q + 2 * e + 1]), cb, a1 * ca);
              nw[e] = pack2<kFmt>(n0, n1);
            }
            reinterpret_cast<uint4*>(orow + c0)[q] = make_uint4(nw[0], nw[1], nw[2], nw[3]);
          }
        }
      }
      if (write && P.pb.lse) P.pb.lse[lidx] = (mx + __log2f(wa + wb)) * kLn2;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

// out = 0, lse = -inf over the computed part (rows no pattern keeps keep them).
template <int kD>
__global__ void __launch_bounds__(256) pp_init_kernel(const Problem pb) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int64_t Nr = pb.q1 - pb.q0, Hr = pb.h1 - pb.h0;
  const int64_t rows = pb.B * Nr * Hr;
  constexpr int kChunks = kD * 2 / 16;  // 16-byte chunks per row
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < rows * kChunks;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int ch = (int)(i % kChunks);
    const int64_t rw = i / kChunks;
    const int64_t h = pb.h0 + rw % Hr, n = pb.q0 + (rw / Hr) % Nr, b = rw / (Hr * Nr);
    reinterpret_cast<uint4*>(static_cast<uint16_t*>(pb.out) + ((b * pb.N + n) * pb.H + h) * kD)[ch] =
        make_uint4(0, 0, 0, 0);
    if (ch == 0 && pb.lse) pb.lse[(b * pb.H + h) * pb.N + n] = -INFINITY;
  }
}

// View [B, N, H, D] (16-bit elements, starting `shift` positions in) as
// (d, h, c, k, b), position = r k + c; boxes of one panel row (64 elements,
// or D below 64) x box_rows k.
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

template <int kFmt, int kD>
int launch_typed(const Problem& pb, cudaStream_t stream) {
  using L = Layout<kD>;
  EncodeTiledFn enc = get_encoder();
  if (!enc) return LONGNET_ERR_CUDA;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  const bool norm = pb.qk_norm != 0;
  auto kernel = norm ? pp_fwd_kernel<kFmt, kD, true> : pp_fwd_kernel<kFmt, kD, false>;
  static bool attr_set[64][2] = {};
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (!attr_set[dev][norm]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmem) != cudaSuccess) {
      cudaGetLastError();
      return LONGNET_ERR_CUDA;
    }
    attr_set[dev][norm] = true;
  }
  int n_sm = 148;
  cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
  {
    const int64_t work = pb.B * (pb.q1 - pb.q0) * (pb.h1 - pb.h0) * (pb.D / 8);
    int64_t blocks = (work + 255) / 256;
    if (blocks > (int64_t)n_sm * 16) blocks = (int64_t)n_sm * 16;
    pp_init_kernel<kD><<<(unsigned)(blocks > 0 ? blocks : 1), 256, 0, stream>>>(pb);
    if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  }
  for (int i = 0; i < pb.n_pat; ++i) {
    Params P;
    memset(&P, 0, sizeof(P));
    P.pb = pb;
    P.p = i;
    P.w = (int)(pb.w[i] < pb.N ? pb.w[i] : pb.N);
    P.r = (int)pb.r[i];
    P.kfull = (int)(pb.N / P.r);
    P.tail = (int)(pb.N % P.r);
    P.r_div = make_fastdiv(P.r);
    P.n_seg = (int)((pb.N + P.w - 1) / P.w);
    P.tiles = (int)(((P.w + P.r - 1) / P.r + kTile - 1) / kTile);
    P.first_call = 0;  // out and lse hold the init values or earlier patterns
    P.scale_log2 = kLog2e / sqrtf((float)pb.D);
    P.wait_limit_ns = kWaitLimitNs;
    Maps maps;
    const void* bases[3] = {pb.q, pb.k, pb.v};
    for (int sh = 0; sh < 2; ++sh)
      for (int t = 0; t < 3; ++t)
        if (!encode(enc, &maps.m[sh][t], bases[t], pb, P.r, sh ? P.tail : 0, P.kfull, t == 0 ? kTile : kBlk))
          return LONGNET_ERR_CUDA;
    const int64_t ctas = pb.B * (pb.h1 - pb.h0) * (int64_t)P.n_seg * P.tiles;
    // programmatic dependent launch: the kernel's CTAs may start while the
    // previous launch on the stream is finishing; each waits for it
    // (griddepcontrol.wait) before it reads or writes out and lse
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)ctas);
    cfg.blockDim = dim3(norm ? kThreadsNorm : kThreads);
    cfg.dynamicSmemBytes = L::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, P, maps) != cudaSuccess) {
      cudaGetLastError();
      return LONGNET_ERR_CUDA;
    }
  }
  return LONGNET_OK;
}

}  // namespace pp

bool perpattern_supports(const Problem& p) {
  if ((p.dtype != LONGNET_DTYPE_BF16 && p.dtype != LONGNET_DTYPE_F16) ||
      (p.D != 16 && p.D != 32 && p.D != 64 && p.D != 128))
    return false;
  if (p.n_pat > 1 && !p.lse) return false;  // the merge runs through lse
  if (p.N > ((int64_t)1 << 30) || p.H > 65535 || p.B > 65535) return false;
  int64_t ctas = 0;
  for (int i = 0; i < p.n_pat; ++i) {
    const int64_t w = p.w[i] < p.N ? p.w[i] : p.N, r = p.r[i];
    if (r > 4096 || p.N / r < 1) return false;
    const int64_t tail = p.N % r;
    // a 128-row box never needs both the first and the last N mod r positions
    if (tail > 0 && p.N < pp::kTile * r + 2 * tail) return false;
    const int64_t c = p.B * (p.h1 - p.h0) * ((p.N + w - 1) / w) * (((w + r - 1) / r + pp::kTile - 1) / pp::kTile);
    if (c > ctas) ctas = c;
  }
  return ctas <= 0x7fffffffLL;
}

int launch_perpattern(const Problem& p, cudaStream_t stream) {
  const bool f16 = p.dtype == LONGNET_DTYPE_F16;
  switch (p.D) {
    case 16:
      return f16 ? pp::launch_typed<tc::kFmtF16, 16>(p, stream) : pp::launch_typed<tc::kFmtBF16, 16>(p, stream);
    case 32:
      return f16 ? pp::launch_typed<tc::kFmtF16, 32>(p, stream) : pp::launch_typed<tc::kFmtBF16, 32>(p, stream);
    case 64:
      return f16 ? pp::launch_typed<tc::kFmtF16, 64>(p, stream) : pp::launch_typed<tc::kFmtBF16, 64>(p, stream);
    default:
      return f16 ? pp::launch_typed<tc::kFmtF16, 128>(p, stream) : pp::launch_typed<tc::kFmtBF16, 128>(p, stream);
  }
}

}  // namespace longnet
