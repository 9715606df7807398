// Kernel family SMALLSEG: the multi-pattern dilated-attention forward when
// every pattern's segments are short (all patterns share one segment length
// W <= 64, bf16 or fp16, D = 64).  Such shapes move far more bytes than they compute
// (the DilatedAttention usage example of the "LongNet" docs page: segment 64,
// dilation 2), so this kernel is built for HBM bandwidth, not tensor peak.
//
// Each pair of warps owns one (batch, segment, head) item at a time, in a
// persistent grid (one CTA per SM, several pairs); the two warps split every
// pattern's 16-row chunks:
//   * three TMA tile loads (Q, K, V: W rows x 128 B, 128-byte swizzle) bring
//     the segment's rows of that head into the pair's shared memory;
//   * every pattern's sparsified segment (head offset o = h mod r, rows
//     o + r*k < W) is read straight from shared memory by ldmatrix (the
//     dilated gather is just a choice of row addresses) and attended with
//     mma.sync m16n8k16 (bf16 or fp16 in, fp32 accumulate) and an fp32 softmax;
//   * patterns other than the r = 1 one park their normalised rows (16-byte
//     chunks rotated by row, like the TMA swizzle, so a fragment's 8 rows hit
//     distinct banks) and lse in the pair's shared memory;
//   * the r = 1 pattern, processed last, merges them row by row with weights
//     e^{lse_p} ("LONGNET: Scaling Transformer to 1 billion tokens", section
//     "Token expansion reaches 1 billion+", read as the softmax-denominator-
//     weighted combination) and the rows go out as coalesced 128-byte stores.
// Pairs of an SM sit at different points of their load/compute/store cycle,
// which keeps bytes in flight while others compute.  The work per item is
// issue-bound (index arithmetic, softmax, mma.sync), so the per-item set-up
// is hoisted and the unmasked case (non-causal, m a multiple of 16) has its
// own instantiation; six pairs leave 168 registers per thread.
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
constexpr int kMaxPat = 4;
constexpr int kMaxPairs = 6;  // 12 warps, 3 per SM sub-partition: up to 168 registers each
constexpr int kTile = kMaxW * kD * 2;  // 8 KB
constexpr int kSmemLimit = 232448;

struct Params {
  Problem pb;
  int W;                    // common segment length
  int order[kMaxPat];       // patterns in processing order (the r = 1 one last)
  int park_off[kMaxPat];    // byte offset of each parked pattern's rows in a pair's region
  int park_rows[kMaxPat];   // rows reserved for it (ceil(W / r))
  int r32[kMaxPat];         // dilations (the host checks they fit)
  uint32_t rcp16[kMaxPat];  // ceil(2^16 / r): (x * rcp16) >> 16 = x / r for 0 <= x < 64
  int pair_bytes;           // shared memory per warp pair (1024-aligned)
  int n_pairs;
  int64_t n_items;          // B * (segments of the part) * (heads of the part)
  uint64_t wait_limit_ns;
};

struct __align__(64) Maps {
  CUtensorMap m[3];  // q, k, v: (d, h, n, b), box (64, 1, W, 1)
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

// ------------------------------------------------------------ kernel

// One 16-row chunk (rows [16 rc, 16 rc + 16) of a sparsified segment with m
// kept rows at o, o + r, ...): S = Q K^T over its m keys, softmax, O = P V,
// normalised.  In the mma fragment layout this lane holds rows g and g + 8 of
// the chunk; their O goes to ov and their lse (log2 domain) to lse0, lse1.
// kMasked: some of the n_kt * 16 key columns are not keys of every row
// (causal, or m not a multiple of 16).
template <int kFmt, bool kMasked>
__device__ __forceinline__ void attend_chunk(uint32_t q_base, uint32_t k_base, uint32_t v_base, int o,
                                             int r, int m, int n_kt, int rc, bool causal,
                                             float scale_log2, int lane, float (&ov)[8][4],
                                             float& lse0, float& lse1) {
  const int g = lane >> 2, t4 = lane & 3;
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  {
    // A fragments address row 16 rc + (lane & 15); B fragments key
    // 16 np + (lane & 7) + 8 (lane >> 4); rows past m are clamped (their
    // results are never used, their keys are masked or absent)
    int qi = rc * 16 + (lane & 15);
    if (qi >= m) qi = m - 1;
    const int qrow = o + r * qi;
    const uint32_t qa = q_base + (uint32_t)qrow * 128u;
    const int qsw = qrow & 7;
    uint32_t ka[4];
    int ksw[4];
#pragma unroll
    for (int np = 0; np < 4; ++np) {
      int kj = np * 16 + (lane & 7) + ((lane >> 4) << 3);
      if (kj >= m) kj = m - 1;
      const int krow = o + r * kj;
      ka[np] = k_base + (uint32_t)krow * 128u;
      ksw[np] = krow & 7;
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
  // ---- softmax over the keys (rows g and g + 8 of this chunk)
  const int row0 = rc * 16 + g, row1 = row0 + 8;
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    if (nt < 2 * n_kt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (kMasked) {
          const int c = nt * 8 + 2 * t4 + e;
          const bool k_ok = c < m;
          if (!(k_ok && (!causal || c <= row0))) acc[nt][e] = -INFINITY;
          if (!(k_ok && (!causal || c <= row1))) acc[nt][2 + e] = -INFINITY;
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
  const float ms0 = mx0 * scale_log2, ms1 = mx1 * scale_log2;  // every row has a key: finite
  float l0 = 0.f, l1 = 0.f;
  uint32_t pa[4][4];  // P as A fragments, one per 16-key step
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    if (nt < 2 * n_kt) {
      float x0, x1, x2, x3;
      f32x2_split(fma_f32x2(f32x2(acc[nt][0], acc[nt][1]), f32x2(scale_log2, scale_log2), f32x2(-ms0, -ms0)), x0, x1);
      f32x2_split(fma_f32x2(f32x2(acc[nt][2], acc[nt][3]), f32x2(scale_log2, scale_log2), f32x2(-ms1, -ms1)), x2, x3);
      const float p0 = ex2(x0), p1 = ex2(x1), p2 = ex2(x2), p3 = ex2(x3);
      l0 += p0 + p1;
      l1 += p2 + p3;
      const int kk = nt >> 1, hi = nt & 1;
      pa[kk][hi * 2 + 0] = pack2<kFmt>(p0, p1);
      pa[kk][hi * 2 + 1] = pack2<kFmt>(p2, p3);
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
      if (vj >= m) vj = m - 1;  // keys past m have P = 0
      const int vrow = o + r * vj;
      const uint32_t va = v_base + (uint32_t)vrow * 128u;
      const int vsw = vrow & 7;
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {  // pairs of 8-dim tiles
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(va + ((uint32_t)((2 * dp + (lane >> 4)) ^ vsw) << 4), b0, b1, b2, b3);
        mma16816<kFmt>(ov[2 * dp], pa[kk], b0, b1);
        mma16816<kFmt>(ov[2 * dp + 1], pa[kk], b2, b3);
      }
    }
  }
  const float inv0 = 1.f / l0, inv1 = 1.f / l1;
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    f32x2_split(mul_f32x2(f32x2(ov[nt][0], ov[nt][1]), f32x2(inv0, inv0)), ov[nt][0], ov[nt][1]);
    f32x2_split(mul_f32x2(f32x2(ov[nt][2], ov[nt][3]), f32x2(inv1, inv1)), ov[nt][2], ov[nt][3]);
  }
  lse0 = ms0 + __log2f(l0);
  lse1 = ms1 + __log2f(l1);
}

template <int kFmt>
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
  uint64_t* bar = reinterpret_cast<uint64_t*>(region + P.pair_bytes - 32);  // TMA landed
  uint64_t* pbar = bar + 1;                                                 // the pair's hand-off
  if (wsub == 0 && lane == 0) {
    mbar_init(bar, 1);
    mbar_init(pbar, 64);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    for (int t = 0; t < 3; ++t)
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.m[t])) : "memory");
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

  const int W = P.W, n_pat = P.pb.n_pat;
  const int H = (int)P.pb.H;
  const int64_t N = P.pb.N;
  const int seg0 = (int)(P.pb.q0 / W), n_seg = (int)((P.pb.q1 - P.pb.q0) / W);
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
    // ---- load the segment's rows of this head (both warps are done with the
    // previous item: the pair synchronised at its end)
    __syncwarp();
    if (wsub == 0 && lane == 0) {
      // the previous item's rows were staged here with ordinary stores
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                   "r"((uint32_t)(3 * W * 128))
                   : "memory");
      tma_load_4d(sQ, &maps.m[0], bar, 0, h, seg * W, b);
      tma_load_4d(sK, &maps.m[1], bar, 0, h, seg * W, b);
      tma_load_4d(sV, &maps.m[2], bar, 0, h, seg * W, b);
    }
    // per-item pattern table: head offset of every pattern, computed once
    int oq[kMaxPat];
#pragma unroll
    for (int pi = 0; pi < kMaxPat; ++pi) oq[pi] = pi < n_pat ? h % P.r32[P.order[pi]] : 0;
    const int64_t row0_pos = (int64_t)b * N + (int64_t)seg * W;  // position of the segment's row 0
    if (!mbar_wait(bar, phase, P.wait_limit_ns)) {
      record_status(P.pb.status, kStatusTimeout);
      // the segment's loads may still be in flight into this pair's shared
      // memory: wait for them once more (bounded) before the warps leave
      mbar_wait(bar, phase, P.wait_limit_ns);
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
      if (!pair_sync()) return;  // every row is normalised before any is read
    }

    bool ok = true;
    for (int pi = 0; pi < n_pat; ++pi) {
      const int p = P.order[pi];
      const bool last = pi == n_pat - 1;
      // the other warp's parked rows are complete before the merging pattern
      if (last && pi > 0 && !(ok = pair_sync())) break;
      const int r = P.r32[p];
      int o = 0;
#pragma unroll
      for (int q = 0; q < kMaxPat; ++q)
        if (q == pi) o = oq[q];
      const int m = o >= W ? 0 : (W - o + r - 1) / r;  // kept rows of this head
      if (m == 0) continue;
      const int n_kt = (m + 15) >> 4;  // 16-key steps
      const bool masked = causal || (m & 15) != 0;
      uint8_t* park = region + P.park_off[p];
      float* park_l = reinterpret_cast<float*>(park + P.park_rows[p] * 128);
      for (int rc = wsub; rc < n_kt; rc += 2) {
        float ov[8][4];
        float lse0, lse1;
        if (masked)
          attend_chunk<kFmt, true>(q_base, k_base, v_base, o, r, m, n_kt, rc, causal, scale_log2, lane, ov, lse0, lse1);
        else
          attend_chunk<kFmt, false>(q_base, k_base, v_base, o, r, m, n_kt, rc, causal, scale_log2, lane, ov, lse0, lse1);
        const int row0 = rc * 16 + g, row1 = row0 + 8;
        if (!last) {
          // ---- park the normalised rows (16-byte chunks rotated by row)
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int row = half ? row1 : row0;
            if (row < m) {
              uint8_t* pr = park + row * 128 + 4 * t4;
#pragma unroll
              for (int nt = 0; nt < 8; ++nt)
                *reinterpret_cast<uint32_t*>(pr + ((nt ^ (row & 7)) << 4)) =
                    pack2<kFmt>(ov[nt][2 * half], ov[nt][2 * half + 1]);
              if (t4 == 0) park_l[row] = half ? lse1 : lse0;
            }
          }
        } else {
          // ---- merge with the parked patterns, stage over the row's own Q row
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int row = half ? row1 : row0;  // sparse index = position in segment (r = 1)
            float lse = half ? lse1 : lse0;
            if (row < m) {
#pragma unroll
              for (int qi = 0; qi < kMaxPat - 1; ++qi) {
                if (qi >= pi) break;
                const int q = P.order[qi];
                const int rq = P.r32[q];
                const int rel = row - oq[qi];
                const int kq = (int)(((uint32_t)rel * P.rcp16[q]) >> 16);  // rel / rq, exact for rel < 64
                if (rel < 0 || kq * rq != rel) continue;
                const uint8_t* pk = region + P.park_off[q];
                const float lq = reinterpret_cast<const float*>(pk + P.park_rows[q] * 128)[kq];
                const float mxl = fmaxf(lse, lq);
                const float wa = ex2(lse - mxl), wb = ex2(lq - mxl);
                const float iw = 1.f / (wa + wb);
                const float ca = wa * iw, cb = wb * iw;
                const uint8_t* pq = pk + kq * 128 + 4 * t4;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                  float plo, phi;
                  unpack2<kFmt>(*reinterpret_cast<const uint32_t*>(pq + ((nt ^ (kq & 7)) << 4)), plo, phi);
                  ov[nt][2 * half] = fmaf(plo, cb, ov[nt][2 * half] * ca);
                  ov[nt][2 * half + 1] = fmaf(phi, cb, ov[nt][2 * half + 1] * ca);
                }
                lse = mxl + __log2f(wa + wb);
              }
              // stage the row over its own Q row (no longer read: later chunks
              // read other rows) in the same swizzled layout
              uint8_t* sr = sQ + row * 128 + 4 * t4;
#pragma unroll
              for (int nt = 0; nt < 8; ++nt)
                *reinterpret_cast<uint32_t*>(sr + ((nt ^ (row & 7)) << 4)) =
                    pack2<kFmt>(ov[nt][2 * half], ov[nt][2 * half + 1]);
              if (t4 == 0 && P.pb.lse)
                P.pb.lse[((int64_t)b * H + h) * N + (int64_t)seg * W + row] = lse * 0.69314718055994531f;
            }
          }
        }
        __syncwarp();
      }
    }
    if (!ok) return;
    // rows this thread wrote with ordinary stores (normalised q and k, staged
    // output) may next be overwritten by the async proxy (the next item's TMA)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    // ---- coalesced store of the rows this warp staged (its 16-row chunks):
    // 16-byte chunks, 8 per row
    __syncwarp();
    {
      uint16_t* out_seg = static_cast<uint16_t*>(P.pb.out) + (row0_pos * H + h) * kD;  // 16-bit elements
      const int64_t row_stride = (int64_t)H * kD;
      for (int rc = wsub; rc * 16 < W; rc += 2) {
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int idx = it * 32 + lane;
          const int row = rc * 16 + (idx >> 3), ch = idx & 7;
          if (row < W) {
            const uint4 u = *reinterpret_cast<const uint4*>(sQ + sw_addr(0, row, ch));
            *reinterpret_cast<uint4*>(out_seg + row * row_stride + ch * 8) = u;
          }
        }
      }
    }
    if (!pair_sync()) return;
  }
}

// ------------------------------------------------------------ host side

// Layout of one warp pair's shared memory for these patterns; 0 if unsupported.
int pair_bytes(const Problem& p, int* park_off, int* park_rows, int* order) {
  int n1 = 0, k = 0;
  for (int i = 0; i < p.n_pat; ++i) {
    if (p.r[i] == 1) ++n1;
  }
  if (n1 != 1) return 0;
  int off = 3 * kTile;
  for (int i = 0; i < p.n_pat; ++i) {
    if (p.r[i] != 1) {
      order[k++] = i;
      park_off[i] = off;
      park_rows[i] = (int)((p.w[0] + p.r[i] - 1) / p.r[i]);
      off += park_rows[i] * 128 + park_rows[i] * 4;
    }
  }
  for (int i = 0; i < p.n_pat; ++i) {
    if (p.r[i] == 1) {
      order[k++] = i;
      park_off[i] = 0;
      park_rows[i] = 0;
    }
  }
  off += 32;                                 // mbarriers
  return (off + 1023) & ~1023;
}

}  // namespace ss

bool smallseg_supports(const Problem& p) {
  using namespace ss;
  if ((p.dtype != LONGNET_DTYPE_BF16 && p.dtype != LONGNET_DTYPE_F16) || p.D != kD) return false;
  if (p.n_pat < 1 || p.n_pat > kMaxPat) return false;
  const int64_t W = p.w[0];
  if (W < 1 || W > kMaxW || W % 8 != 0) return false;
  for (int i = 0; i < p.n_pat; ++i)
    if (p.w[i] != W) return false;
  if (W > p.N || p.N % W != 0) return false;  // whole segments only
  if (p.q0 % W != 0 || p.q1 % W != 0) return false;  // a part of whole segments
  if (p.H > 65535 || p.B > 65535 || p.N > (int64_t)INT32_MAX) return false;
  for (int i = 0; i < p.n_pat; ++i)
    if (p.r[i] < 1 || p.r[i] > (int64_t)INT32_MAX) return false;
  int off[kMaxPat], rows[kMaxPat], order[kMaxPat];
  const int pb = pair_bytes(p, off, rows, order);
  return pb > 0 && pb + 1024 <= kSmemLimit;
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
  P.pair_bytes = pair_bytes(pb, P.park_off, P.park_rows, P.order);
  for (int i = 0; i < pb.n_pat; ++i) {
    P.r32[i] = (int)pb.r[i];
    P.rcp16[i] = (uint32_t)((65536 + pb.r[i] - 1) / pb.r[i]);
  }
  if (P.pair_bytes <= 0) return LONGNET_ERR_UNSUPPORTED;
  P.n_pairs = (kSmemLimit - 1024) / P.pair_bytes;
  if (P.n_pairs > kMaxPairs) P.n_pairs = kMaxPairs;
  if (P.n_pairs < 1) return LONGNET_ERR_UNSUPPORTED;
  // items of the computed part: (b, segment, head) with segments in
  // [q0 / W, q1 / W) and heads in [h0, h1)
  P.n_items = pb.B * ((pb.q1 - pb.q0) / P.W) * (pb.h1 - pb.h0);
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
    int64_t B, N, H, W, dtype;
  };
  static MapKey last[64] = {};
  static Maps last_maps[64];
  const MapKey key{pb.q, pb.k, pb.v, pb.B, pb.N, pb.H, P.W, pb.dtype};
  if (memcmp(&last[dev], &key, sizeof(key)) == 0) {
    maps = last_maps[dev];
  } else {
    last[dev] = MapKey{};
    const void* bases[3] = {pb.q, pb.k, pb.v};
    for (int t = 0; t < 3; ++t) {
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
  auto kernel = f16 ? smallseg_kernel<kFmtF16> : smallseg_kernel<kFmtBF16>;
  static bool attr_set[64][2] = {};
  if (!attr_set[dev][f16]) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) != cudaSuccess)
      return LONGNET_ERR_CUDA;
    attr_set[dev][f16] = true;
  }
  const int smem = P.n_pairs * P.pair_bytes + 1024;
  int64_t grid = (P.n_items + P.n_pairs - 1) / P.n_pairs;
  if (grid > n_sm) grid = n_sm;
  kernel<<<(unsigned)grid, P.n_pairs * 64, smem, stream>>>(P, maps);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

}  // namespace longnet
