// Kernel family SMALLSEG: the multi-pattern dilated-attention forward when
// every pattern's segments are short (all patterns share one segment length
// W <= 64, bf16 or fp16, D = 64; the last segment may be the shorter rest of
// the sequence).  Such shapes move far more bytes than they compute
// (the DilatedAttention usage example of the "LongNet" docs page: segment 64,
// dilation 2), so this kernel is built for HBM bandwidth, not tensor peak.
//
// One softmax per segment.  With a common segment length, every pattern's
// sparsified segment of head h is a subset of the same W positions: pattern
// p keeps the positions i = o_p (mod r_p), o_p = h mod r_p.  Combining the
// patterns' outputs with weights equal to their softmax denominators
// ("LONGNET: Scaling Transformer to 1 billion tokens", section "Token
// expansion reaches 1 billion+", read as the denominator-weighted
// combination) gives, for a row i,
//     out_i = sum_j c_ij e^{s_ij} v_j / sum_j c_ij e^{s_ij},
//     c_ij  = #{p : i and j both kept by p}   (and j <= i when causal),
// and the combined lse is log sum_j c_ij e^{s_ij}: the patterns' numerators
// and denominators simply add.  So one Q K^T over the segment, one softmax
// whose exponent carries log2 c_ij, and one P V replace the per-pattern
// passes and their merge; no partial result is rounded or parked.
//
// Each pair of warps owns one (batch, segment, head) item at a time, in a
// persistent grid (one CTA per SM, several pairs); the two warps split the
// segment's 16-row chunks:
//   * three TMA tile loads (Q, K, V: W rows x 128 B, 128-byte swizzle) bring
//     the segment's rows of that head into the pair's shared memory;
//   * S = Q K^T and O = P V by mma.sync m16n8k16 (bf16 or fp16 in, fp32
//     accumulate) on ldmatrix fragments, fp32 softmax with exp2;
//   * the weights: in the accumulator layout a lane holds rows g, g + 8 and
//     columns 8 nt + 2 t4 + {0, 1}; when every r divides 8 these are the same
//     residues mod r for every chunk and every nt, so log2 c is one packed
//     pair per lane, read from a table indexed by h mod 8 and the lane (the
//     exponent costs nothing extra).  Other dilations take a general variant
//     that counts c per element from per-pattern bit masks;
//   * the normalised rows are staged over the rows' own Q rows (same swizzled
//     layout) and leave by one TMA tile store per item.
// Pairs of an SM sit at different points of their load/compute/store cycle,
// which keeps bytes in flight while others compute; each pair also has its
// next item's tiles brought into L2 (TMA prefetch) when it loads the current
// one, so the next loads wait for L2, not HBM.
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
#include "tc_ptx.cuh"  // the tensor-map encoder lookup

namespace longnet {
namespace ss {

constexpr int kD = 64;
constexpr int kMaxW = 64;
constexpr int kMaxPat = 8;         // patterns when every r divides 8
constexpr int kMaxPatGeneral = 4;  // patterns otherwise (per-pattern masks per lane)
constexpr int kMaxPairs = 6;       // 12 warps, 3 per SM sub-partition: up to 168 registers each
constexpr int kTile = kMaxW * kD * 2;  // 8 KB
constexpr int kSmemLimit = 232448;
constexpr int kTableBytes = 8 * 32 * 8;  // [h mod 8][lane] packed log2 c pair

// Softmax variants.
//   kModeFull:    every r divides 8, some r = 1, not causal, W a multiple of 16:
//                 every key of every row has weight >= 1, no column is masked
//                 (but the keys past the end of a short last segment);
//   kModeMasked:  every r divides 8, otherwise (causal, W not a multiple of
//                 16, or keys of weight 0);
//   kModeGeneral: some r does not divide 8: weights counted per element.
constexpr int kModeFull = 0, kModeMasked = 1, kModeGeneral = 2;

struct Params {
  Problem pb;
  int W;                  // common segment length
  int r32[kMaxPat];       // dilations (the host checks they fit)
  int pair_bytes;         // shared memory per warp pair (1024-aligned)
  int n_pairs;
  int64_t n_items;        // B * (segments of the part) * (heads of the part)
  uint64_t wait_limit_ns;
};

struct __align__(64) Maps {
  CUtensorMap m[4];  // q, k, v, out: (d, h, n, b), box (64, 1, W, 1)
};

// ------------------------------------------------------------ PTX helpers

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// Element formats of the 16-bit operands.
constexpr int kFmtF16 = 0, kFmtBF16 = 1;
// D += A * B, m16n8k16, 16-bit inputs (bf16 or f16), fp32 accumulators
template <int kFmt>
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  if constexpr (kFmt == kFmtBF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}
// Two floats rounded to the element format, lo in the low half.
template <int kFmt>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (kFmt == kFmtBF16) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
}
// The two elements of a packed pair as floats (exact).
template <int kFmt>
__device__ __forceinline__ void unpack2(uint32_t u, float& lo, float& hi) {
  if constexpr (kFmt == kFmtBF16) {
    lo = __uint_as_float(u << 16);
    hi = __uint_as_float(u & 0xffff0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&u));
    lo = f.x;
    hi = f.y;
  }
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two fp32 values in one 64-bit register pair, for the packed f32x2 ops.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_split(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Byte address of the 16-byte chunk `ch` of row `row` in a 128-byte-swizzled
// tile of 128-byte rows (the layout the TMA writes).
__device__ __forceinline__ uint32_t sw_addr(uint32_t base, int row, int ch) {
  return base + (uint32_t)row * 128u + ((uint32_t)(ch ^ (row & 7)) << 4);
}

__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int c0, int c1, int c2,
                                             int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// The issuing thread's bulk stores have finished reading shared memory.
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// The issuing thread's bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Brings a tile into L2 (no shared-memory destination, no completion).
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// ------------------------------------------------------------ kernel

// One 16-row chunk (segment rows [16 rc, 16 rc + 16)) against the segment's W
// keys: S = Q K^T, the weighted softmax, O = P V, normalised.  In the mma
// fragment layout this lane holds rows g and g + 8 of the chunk and key
// columns 8 nt + 2 t4 + {0, 1}; their O goes to ov and their lse (log2
// domain, -inf for a row no pattern keeps) to lse0, lse1.
//   kModeFull / kModeMasked: lb = (log2 c, log2 c) of this lane's two key
//     parities (-inf for weight 0), the same for both rows;
//   kModeGeneral: cw0, cw1 = the weights of the lane's 16 key columns for
//     rows g and g + 8, one nibble per column (nibble 2 nt + e).
template <int kFmt, int kMode>
__device__ __forceinline__ void attend_chunk(uint32_t q_base, uint32_t k_base, uint32_t v_base, int W, int n_kt,
                                             int rc, bool causal, float scale_log2, int lane, float2 lb,
                                             uint64_t cw0, uint64_t cw1, float (&ov)[8][4], float& lse0,
                                             float& lse1) {
  const int g = lane >> 2, t4 = lane & 3;
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  {
    // A fragments address row 16 rc + (lane & 15); B fragments key
    // 16 np + (lane & 7) + 8 (lane >> 4); rows and keys past W are clamped
    // (their results are never used, their keys are masked or absent)
    int qi = rc * 16 + (lane & 15);
    if (qi >= W) qi = W - 1;
    const uint32_t qa = q_base + (uint32_t)qi * 128u;
    const int qsw = qi & 7;
    uint32_t ka[4];
    int ksw[4];
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      int kj = np * 16 + (lane & 7) + ((lane >> 4) << 3);
      if (kj >= W) kj = W - 1;
      ka[np] = k_base + (uint32_t)kj * 128u;
      ksw[np] = kj & 7;
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      ldsm_x4(qa + ((uint32_t)((2 * kk + (lane >> 4)) ^ qsw) << 4), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        if (np < n_kt) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(ka[np] + ((uint32_t)((2 * kk + ((lane >> 3) & 1)) ^ ksw[np]) << 4), b0, b1, b2, b3);
          mma16816<kFmt>(acc[2 * np], a, b0, b1);
          mma16816<kFmt>(acc[2 * np + 1], a, b2, b3);
        }
      }
    }
  }
  // ---- weighted softmax over the keys (rows g and g + 8 of this chunk)
  const int row0 = rc * 16 + g, row1 = row0 + 8;
  float l0 = 0.f, l1 = 0.f;
  float m0, m1;  // the exponents' stabilisers (log2 domain)
  uint32_t pa[4][4];  // P as A fragments, one per 16-key step
  if constexpr (kMode == kModeFull) {
    if (W & 15) {
      // a short last segment: the keys past its end (zeros from the load)
      // inside the last 16-key step get no weight
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e)
          if (nt * 8 + 2 * t4 + e >= W) acc[nt][e] = acc[nt][2 + e] = -INFINITY;
    }
    // every weight >= 1: the largest raw score of the row stabilises
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      if (nt < 2 * n_kt) {
        mx0 = fmaxf(mx0, fmaxf(acc[nt][0], acc[nt][1]));
        mx1 = fmaxf(mx1, fmaxf(acc[nt][2], acc[nt][3]));
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    m0 = mx0 * scale_log2;
    m1 = mx1 * scale_log2;
    // p = 2^(s * scale + log2 c - m) = c 2^(s * scale - m) <= c
    const uint64_t sc2 = f32x2(scale_log2, scale_log2);
    const uint64_t a0 = f32x2(lb.x - m0, lb.y - m0), a1 = f32x2(lb.x - m1, lb.y - m1);
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      if (nt < 2 * n_kt) {
        float x0, x1, x2, x3;
        f32x2_split(fma_f32x2(f32x2(acc[nt][0], acc[nt][1]), sc2, a0), x0, x1);
        f32x2_split(fma_f32x2(f32x2(acc[nt][2], acc[nt][3]), sc2, a1), x2, x3);
        const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
        l0 += p0 + p1;
        l1 += p2 + p3;
        const int kk = nt >> 1, hi = nt & 1;
        pa[kk][hi * 2 + 0] = pack2<kFmt>(p0, p1);
        pa[kk][hi * 2 + 1] = pack2<kFmt>(p2, p3);
      }
    }
  } else {
    // x = s * scale + log2 c, -inf where the key is past W, after the row
    // (causal) or of weight 0; the row's largest x stabilises
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      if (nt < 2 * n_kt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = nt * 8 + 2 * t4 + e;
          const bool ok0 = c < W && (!causal || c <= row0);
          const bool ok1 = c < W && (!causal || c <= row1);
          if constexpr (kMode == kModeMasked) {
            const float b = e ? lb.y : lb.x;
            acc[nt][e] = ok0 ? fmaf(acc[nt][e], scale_log2, b) : -INFINITY;
            acc[nt][2 + e] = ok1 ? fmaf(acc[nt][2 + e], scale_log2, b) : -INFINITY;
          } else {
            const int sh = 4 * (2 * nt + e);
            const bool w0 = ((cw0 >> sh) & 15u) != 0, w1 = ((cw1 >> sh) & 15u) != 0;
            acc[nt][e] = ok0 && w0 ? acc[nt][e] * scale_log2 : -INFINITY;
            acc[nt][2 + e] = ok1 && w1 ? acc[nt][2 + e] * scale_log2 : -INFINITY;
          }
          mx0 = fmaxf(mx0, acc[nt][e]);
          mx1 = fmaxf(mx1, acc[nt][2 + e]);
        }
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    // a row with no key of positive weight (no pattern keeps it) has mx =
    // -inf: any finite stabiliser gives p = 0 and l = 0
    m0 = mx0 == -INFINITY ? 0.f : mx0;
    m1 = mx1 == -INFINITY ? 0.f : mx1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      if (nt < 2 * n_kt) {
        float p0 = ex2(acc[nt][0] - m0), p1 = ex2(acc[nt][1] - m0);
        float p2 = ex2(acc[nt][2] - m1), p3 = ex2(acc[nt][3] - m1);
        if constexpr (kMode == kModeGeneral) {
          // times the weight (a nibble, as float through the 2^23 magic number)
          const int sh = 4 * (2 * nt);
          auto wf = [](uint64_t w, int s) {
            return __uint_as_float(0x4B000000u | (uint32_t)((w >> s) & 15u)) - 8388608.f;
          };
          p0 *= wf(cw0, sh);
          p1 *= wf(cw0, sh + 4);
          p2 *= wf(cw1, sh);
          p3 *= wf(cw1, sh + 4);
        }
        l0 += p0 + p1;
        l1 += p2 + p3;
        const int kk = nt >> 1, hi = nt & 1;
        pa[kk][hi * 2 + 0] = pack2<kFmt>(p0, p1);
        pa[kk][hi * 2 + 1] = pack2<kFmt>(p2, p3);
      }
    }
  }
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  // ---- O = P V (16 rows x 64 dims)
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) ov[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    if (kk < n_kt) {
      int vj = kk * 16 + (lane & 15);
      if (vj >= W) vj = W - 1;  // keys past W have P = 0
      const uint32_t va = v_base + (uint32_t)vj * 128u;
      const int vsw = vj & 7;
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {  // pairs of 8-dim tiles
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(va + ((uint32_t)((2 * dp + (lane >> 4)) ^ vsw) << 4), b0, b1, b2, b3);
        mma16816<kFmt>(ov[2 * dp], pa[kk], b0, b1);
        mma16816<kFmt>(ov[2 * dp + 1], pa[kk], b2, b3);
      }
    }
  }
  if constexpr (kMode == kModeFull) {
    // l >= 1: the row's largest score has weight >= 1 and exponent >= 0
    const float inv0 = 1.f / l0, inv1 = 1.f / l1;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      f32x2_split(mul_f32x2(f32x2(ov[nt][0], ov[nt][1]), f32x2(inv0, inv0)), ov[nt][0], ov[nt][1]);
      f32x2_split(mul_f32x2(f32x2(ov[nt][2], ov[nt][3]), f32x2(inv1, inv1)), ov[nt][2], ov[nt][3]);
    }
    lse0 = m0 + __log2f(l0);
    lse1 = m1 + __log2f(l1);
  } else {
    // a row no pattern keeps: out = 0, lse = -inf
    const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      f32x2_split(mul_f32x2(f32x2(ov[nt][0], ov[nt][1]), f32x2(inv0, inv0)), ov[nt][0], ov[nt][1]);
      f32x2_split(mul_f32x2(f32x2(ov[nt][2], ov[nt][3]), f32x2(inv1, inv1)), ov[nt][2], ov[nt][3]);
    }
    lse0 = l0 > 0.f ? m0 + __log2f(l0) : -INFINITY;
    lse1 = l1 > 0.f ? m1 + __log2f(l1) : -INFINITY;
  }
}

// Pattern (r, o)'s mask of this lane's 16 key columns: nibble 2 nt + e is 1
// when column 8 nt + 2 t4 + e = o (mod r).
__device__ __forceinline__ uint64_t column_nibbles(int r, int o, int t4) {
  uint64_t w = 0;
  const int step = 8 % r;
  int m0 = (2 * t4) % r, m1 = (2 * t4 + 1) % r;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    w |= (uint64_t)(m0 == o) << (4 * (2 * nt));
    w |= (uint64_t)(m1 == o) << (4 * (2 * nt + 1));
    m0 += step;
    m0 -= m0 >= r ? r : 0;
    m1 += step;
    m1 -= m1 >= r ? r : 0;
  }
  return w;
}
// Weight nibbles of this lane's key columns for `row`: the sum of the column
// masks of the patterns keeping the row (c = #{p : row = o_p and
// column = o_p (mod r_p)}).
__device__ __forceinline__ uint64_t weight_nibbles(int row, int n_pat, const int* rp, const int* op,
                                                   const uint64_t* cols) {
  uint64_t w = 0;
#pragma unroll
  for (int p = 0; p < kMaxPatGeneral; ++p)
    if (p < n_pat && row % rp[p] == op[p]) w += cols[p];
  return w;
}

template <int kFmt, int kMode>
__global__ void __launch_bounds__(kMaxPairs * 64, 1)
    smallseg_kernel(const __grid_constant__ Params P, const __grid_constant__ Maps maps) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = warp >> 1, wsub = warp & 1;
  uint8_t* region = smem + (size_t)pair * P.pair_bytes;
  uint8_t* sQ = region;
  uint8_t* sK = region + kTile;
  uint8_t* sV = region + 2 * kTile;
  uint64_t* bar = reinterpret_cast<uint64_t*>(region + 3 * kTile);  // TMA landed
  uint64_t* pbar = bar + 1;                                         // the pair's hand-off
  float2* wtab = reinterpret_cast<float2*>(smem + (size_t)P.n_pairs * P.pair_bytes);  // [h mod 8][lane]
  const int n_pat = P.pb.n_pat;
  if (wsub == 0 && lane == 0) {
    mbar_init(bar, 1);
    mbar_init(pbar, 64);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int t = 0; t < 4; ++t)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.m[t])) : "memory");
  }
  if constexpr (kMode != kModeGeneral) {
    // log2 of the weights of a lane's two key parities, for each h mod 8:
    // rows g (and g + 8, 16 rc + g) and columns 2 t4 + e (+ 8 nt) have the
    // same residues mod every r dividing 8
    for (int i = threadIdx.x; i < 8 * 32; i += blockDim.x) {
      const int hc = i >> 5, g = (i & 31) >> 2, t4 = i & 3;
      int c[2] = {0, 0};
      for (int p = 0; p < n_pat; ++p) {
        const int r = P.r32[p], o = hc % r;
        if (g % r != o) continue;
        c[0] += (2 * t4) % r == o;
        c[1] += (2 * t4 + 1) % r == o;
      }
      wtab[i] = make_float2(c[0] ? log2f((float)c[0]) : -INFINITY, c[1] ? log2f((float)c[1]) : -INFINITY);
    }
  }
  __syncthreads();
  uint32_t pphase = 0;
  // Bounded barrier of the warp pair (both warps arrive, both wait).
  auto pair_sync = [&]() -> bool {
    mbar_arrive_cta(pbar);
    const bool ok = mbar_wait(pbar, pphase, P.wait_limit_ns);
    pphase ^= 1;
    if (!ok) record_status(P.pb.status, kStatusTimeout);
    return ok;
  };
  const bool issuer = wsub == 0 && lane == 0;  // TMA loads and the bulk store of the pair

  const int W = P.W;
  const int H = (int)P.pb.H;
  const int64_t N = P.pb.N;
  // segments of the part; the last one may be the shorter rest of the sequence
  const int seg0 = (int)(P.pb.q0 / W), n_seg = (int)((P.pb.q1 - P.pb.q0 + W - 1) / W);
  const int h0 = (int)P.pb.h0, Hr = (int)(P.pb.h1 - P.pb.h0);
  const bool causal = P.pb.causal != 0;
  const int g = lane >> 2, t4 = lane & 3;  // mma fragment coordinates
  const float scale_log2 = 1.4426950408889634f * rsqrtf((float)kD);
  const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
  uint32_t phase = 0;

  for (int64_t item = (int64_t)blockIdx.x * P.n_pairs + pair; item < P.n_items;
       item += (int64_t)gridDim.x * P.n_pairs, phase ^= 1) {
    const int h = h0 + (int)(item % Hr);
    const int64_t bs = item / Hr;
    const int seg = seg0 + (int)(bs % n_seg);
    const int b = (int)(bs / n_seg);
    // rows (and keys) of this segment: W, or the rest of the sequence; the
    // tiles' rows past N load as zeros and are not stored
    const int Wr = N - (int64_t)seg * W < W ? (int)(N - (int64_t)seg * W) : W;
    const int n_kt = (Wr + 15) >> 4;  // 16-key steps and 16-row chunks
    // ---- load the segment's rows of this head (both warps are done with the
    // previous item: the pair synchronised before its store)
    __syncwarp();
    if (issuer) {
      // the previous item's store has read the staged rows out of sQ, and
      // rows written with ordinary stores are ordered before the async proxy
      bulk_wait_read();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                   "r"((uint32_t)(3 * W * 128))
                   : "memory");
      tma_load_4d(sQ, &maps.m[0], bar, 0, h, seg * W, b);
      tma_load_4d(sK, &maps.m[1], bar, 0, h, seg * W, b);
      tma_load_4d(sV, &maps.m[2], bar, 0, h, seg * W, b);
      // this pair's next item into L2, so that its loads find it there
      const int64_t nx = item + (int64_t)gridDim.x * P.n_pairs;
      if (nx < P.n_items) {
        const int hn = h0 + (int)(nx % Hr);
        const int64_t bsn = nx / Hr;
        const int segn = seg0 + (int)(bsn % n_seg), bn = (int)(bsn / n_seg);
        for (int t = 0; t < 3; ++t) tma_prefetch_4d(&maps.m[t], 0, hn, segn * W, bn);
      }
    }
    float2 lb = make_float2(0.f, 0.f);
    int op[kMaxPatGeneral];
    uint64_t cols[kMaxPatGeneral];
    if constexpr (kMode != kModeGeneral) {
      lb = wtab[(h & 7) * 32 + lane];
    } else {
#pragma unroll
      for (int p = 0; p < kMaxPatGeneral; ++p) {
        op[p] = p < n_pat ? h % P.r32[p] : 0;
        cols[p] = p < n_pat ? column_nibbles(P.r32[p], op[p], t4) : 0;
      }
    }
    if (!mbar_wait(bar, phase, P.wait_limit_ns)) {
      record_status(P.pb.status, kStatusTimeout);
      // the segment's loads may still be in flight into this pair's shared
      // memory: wait for them once more (bounded) before the warps leave
      mbar_wait(bar, phase, P.wait_limit_ns);
      if (issuer) bulk_wait_all();
      return;
    }
    if (P.pb.qk_norm) {
      // q and k rows to unit L2 norm (x / max(|x|, 1e-12), fp32), rounded back
      // to the input format in place; the pair splits the 2W rows
      for (int rr = wsub * 32 + lane; rr < 2 * W; rr += 64) {
        uint8_t* tile = rr < W ? sQ : sK;
        const int row = rr < W ? rr : rr - W;
        uint4 u[8];
        float ss = 0.f;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          u[ch] = *reinterpret_cast<const uint4*>(tile + sw_addr(0, row, ch));
          const uint32_t wv[4] = {u[ch].x, u[ch].y, u[ch].z, u[ch].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float lo, hi;
            unpack2<kFmt>(wv[e], lo, hi);
            ss = fmaf(lo, lo, fmaf(hi, hi, ss));
          }
        }
        const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t wv[4] = {u[ch].x, u[ch].y, u[ch].z, u[ch].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            float lo, hi;
            unpack2<kFmt>(wv[e], lo, hi);
            wv[e] = pack2<kFmt>(lo * inv, hi * inv);
          }
          *reinterpret_cast<uint4*>(tile + sw_addr(0, row, ch)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
      }
      if (!pair_sync()) {  // every row is normalised before any is read
        if (issuer) bulk_wait_all();
        return;
      }
    }

    const int64_t seg_pos = (int64_t)seg * W;  // position of the segment's row 0
    for (int rc = wsub; rc < n_kt; rc += 2) {
      uint64_t cw0 = 0, cw1 = 0;
      if constexpr (kMode == kModeGeneral) {
        cw0 = weight_nibbles(rc * 16 + g, n_pat, P.r32, op, cols);
        cw1 = weight_nibbles(rc * 16 + g + 8, n_pat, P.r32, op, cols);
      }
      float ov[8][4];
      float lse0, lse1;
      attend_chunk<kFmt, kMode>(q_base, k_base, v_base, Wr, n_kt, rc, causal, scale_log2, lane, lb, cw0, cw1, ov,
                                lse0, lse1);
      // ---- stage the rows over their own Q rows (no longer read: later
      // chunks read other rows) in the same swizzled layout
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int row = rc * 16 + g + 8 * half;
        if (row < Wr) {
          uint8_t* sr = sQ + row * 128 + 4 * t4;
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
            *reinterpret_cast<uint32_t*>(sr + ((nt ^ (row & 7)) << 4)) =
                pack2<kFmt>(ov[nt][2 * half], ov[nt][2 * half + 1]);
          if (t4 == 0 && P.pb.lse)
            P.pb.lse[((int64_t)b * H + h) * N + seg_pos + row] = (half ? lse1 : lse0) * 0.69314718055994531f;
        }
      }
    }
    // staged rows (and normalised q and k) are ordered before the async
    // proxy's store and the next item's loads
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (!pair_sync()) {
      if (issuer) bulk_wait_all();
      return;
    }
    if (issuer) tma_store_4d(&maps.m[3], sQ, 0, h, seg * W, b);
  }
  if (issuer) bulk_wait_all();
}

// ------------------------------------------------------------ host side

namespace {
bool divides8(int64_t r) { return r == 1 || r == 2 || r == 4 || r == 8; }
}  // namespace

// Shared memory of one warp pair: Q, K, V tiles and two mbarriers.
constexpr int kPairBytes = (3 * kTile + 16 + 1023) & ~1023;

}  // namespace ss

bool smallseg_supports(const Problem& p) {
  using namespace ss;
  if ((p.dtype != LONGNET_DTYPE_BF16 && p.dtype != LONGNET_DTYPE_F16) || p.D != kD) return false;
  if (p.n_pat < 1 || p.n_pat > kMaxPat) return false;
  bool general = false;
  for (int i = 0; i < p.n_pat; ++i) general |= !divides8(p.r[i]);
  if (general && p.n_pat > kMaxPatGeneral) return false;
  const int64_t W = p.w[0];
  if (W < 1 || W > kMaxW || W % 8 != 0) return false;
  for (int i = 0; i < p.n_pat; ++i)
    if (p.w[i] != W) return false;
  // a part of whole segments (the sequence's last one may be shorter)
  if (p.q0 % W != 0 || (p.q1 % W != 0 && p.q1 != p.N)) return false;
  if (p.H > 65535 || p.B > 65535 || p.N > (int64_t)INT32_MAX) return false;
  for (int i = 0; i < p.n_pat; ++i)
    if (p.r[i] < 1 || p.r[i] > (int64_t)INT32_MAX) return false;
  // the tensor maps' base addresses (the strides are multiples of 128 B)
  const void* ptrs[4] = {p.q, p.k, p.v, p.out};
  for (const void* ptr : ptrs)
    if (reinterpret_cast<uintptr_t>(ptr) % 16 != 0) return false;
  return true;
}

int launch_smallseg(const Problem& pb, cudaStream_t stream) {
  using namespace ss;
  tc::EncodeTiledFn enc = tc::get_encoder();
  if (!enc) return LONGNET_ERR_CUDA;
  static Params P;
  static Maps maps;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  memset(&P, 0, sizeof(P));
  P.pb = pb;
  P.W = (int)pb.w[0];
  P.wait_limit_ns = kWaitLimitNs;
  P.pair_bytes = kPairBytes;
  bool general = false, has_r1 = false;
  for (int i = 0; i < pb.n_pat; ++i) {
    P.r32[i] = (int)pb.r[i];
    general |= !divides8(pb.r[i]);
    has_r1 |= pb.r[i] == 1;
  }
  P.n_pairs = (kSmemLimit - 1024 - kTableBytes) / P.pair_bytes;
  if (P.n_pairs > kMaxPairs) P.n_pairs = kMaxPairs;
  // items of the computed part: (b, segment, head) with segments in
  // [q0 / W, q1 / W) and heads in [h0, h1)
  P.n_items = pb.B * ((pb.q1 - pb.q0 + P.W - 1) / P.W) * (pb.h1 - pb.h0);
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return LONGNET_ERR_CUDA;
  // The tensor maps of the last call on each device are reused while the
  // tensors and their shape stay the same.
  struct MapKey {
    const void* q;
    const void* k;
    const void* v;
    const void* out;
    int64_t B, N, H, W, dtype;
  };
  static MapKey last[64] = {};
  static Maps last_maps[64];
  const MapKey key{pb.q, pb.k, pb.v, pb.out, pb.B, pb.N, pb.H, P.W, pb.dtype};
  if (memcmp(&last[dev], &key, sizeof(key)) == 0) {
    maps = last_maps[dev];
  } else {
    last[dev] = MapKey{};
    const void* bases[4] = {pb.q, pb.k, pb.v, pb.out};
    for (int t = 0; t < 4; ++t) {
      cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)pb.H, (cuuint64_t)pb.N, (cuuint64_t)pb.B};
      cuuint64_t strides[3] = {(cuuint64_t)(kD * 2), (cuuint64_t)(pb.H * kD * 2),
                               (cuuint64_t)(pb.N * pb.H * kD * 2)};
      cuuint32_t box[4] = {(cuuint32_t)kD, 1, (cuuint32_t)P.W, 1};
      cuuint32_t estr[4] = {1, 1, 1, 1};
      if (enc(&maps.m[t], pb.dtype == LONGNET_DTYPE_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(bases[t]), dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return LONGNET_ERR_CUDA;
    }
    last_maps[dev] = maps;
    last[dev] = key;
  }
  const bool f16 = pb.dtype == LONGNET_DTYPE_F16;
  const int mode = general ? kModeGeneral
                   : (has_r1 && !pb.causal && P.W % 16 == 0) ? kModeFull
                                                               : kModeMasked;
  using KernelFn = void (*)(Params, Maps);
  static const KernelFn kernels[2][3] = {
      {smallseg_kernel<kFmtF16, kModeFull>, smallseg_kernel<kFmtF16, kModeMasked>,
       smallseg_kernel<kFmtF16, kModeGeneral>},
      {smallseg_kernel<kFmtBF16, kModeFull>, smallseg_kernel<kFmtBF16, kModeMasked>,
       smallseg_kernel<kFmtBF16, kModeGeneral>}};
  const KernelFn kernel = kernels[f16 ? 0 : 1][mode];
  static bool attr_set[64][2][3] = {};
  if (!attr_set[dev][f16][mode]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
      return LONGNET_ERR_CUDA;
    attr_set[dev][f16][mode] = true;
  }
  const int smem = P.n_pairs * P.pair_bytes + kTableBytes + 1024;
  int64_t grid = (P.n_items + P.n_pairs - 1) / P.n_pairs;
  if (grid > n_sm) grid = n_sm;
  kernel<<<(unsigned)grid, P.n_pairs * 64, smem, stream>>>(P, maps);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

}  // namespace longnet
