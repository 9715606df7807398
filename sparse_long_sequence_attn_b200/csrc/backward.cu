// Backward of the multi-pattern dilated-attention forward: dq, dk, dv.
//
// The pages present LongNet as a model to train ("LONGNET: Scaling
// Transformer to 1 billion tokens", section "Distributed training"; "LongNet"
// docs page, features list), so the gradient of the forward is the step after
// it.  The forward's combination of patterns weighted by e^{lse_p} is one
// softmax over every (pattern, key) pair that reaches a row (a key kept by two
// patterns counts twice), so its gradient is that of a single softmax over the
// same pairs: with P_ij = e^{s_ij - lse_i} (lse_i the combined lse the forward
// saved), delta_i = <dout_i, out_i> and ds_ij = P_ij (<dout_i, v_j> - delta_i),
//   dq_i = sum_j ds_ij k_j / sqrt(D),  dk_j = sum_i ds_ij q_i / sqrt(D),
//   dv_j = sum_i P_ij dout_i,
// each sum running over the pairs (i, j) of every pattern that keeps both rows.
//
// The gradients are written in fp32 whatever the input format.  Two families:
//
// SIMT (any D in {16, 32, 64, 128}, every dtype): two fp32 kernels, one warp
// per row, each writing only its own rows (no atomics):
//   - dq: the row as a query, over the keys of every pattern keeping it (the
//     forward SIMT kernel's walk), recomputing P from q, k and the saved lse;
//   - dk, dv: the row as a key, over the queries of every pattern keeping it
//     (the ones at or after it when causal), recomputing P and delta_i from
//     q, dout, out and lse of each query.
//
// Tiles (bf16 or fp16, D = 64): the tensor-core path.  Work is cut per
// (pattern, batch, head, segment) into 64-row tiles of the sparsified segment,
// gathered row by row from [B, N, H, D] (position first + r * t for kept row
// t) with cp.async into 128-byte-swizzled shared-memory tiles.  Per tile pair
// the five products (S, dP, dV, dK, dQ) run on mma.sync m16n8k16 with fp32
// accumulators; P and dS go from accumulator registers straight into the next
// product's A operand.  Two kernels, so that no tile pair needs atomics:
//   - dk, dv: a CTA owns a key tile and walks the query tiles that reach it,
//     keeping dK and dV in registers;
//   - dq: a CTA owns a query tile and walks its key tiles, keeping dQ.
// S and dP are computed in both (7 products per tile pair instead of 5).  A
// row kept by several patterns gets one fp32 atomic add per pattern, at the
// end of the owning CTA; the call zeroes the gradients first.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "device_util.cuh"
#include "params.h"

namespace longnet {
namespace {

constexpr int kBwdWarps = 4;

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld(const __half* p) { return __half2float(*p); }

__device__ __forceinline__ float warp_sum32(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Back through the qk_norm normalisation xhat = a x, a = 1 / max(|x|, 1e-12):
// given the cotangent g of xhat (lane l holds dims l, l + 32, ...), the
// cotangent of x is a (g - xhat <xhat, g>) where |x| > 1e-12, else a g.
// xhat: the normalised row in shared memory; xx = |x|^2.
template <int D>
__device__ __forceinline__ void project_row(float (&g)[(D + 31) / 32], const float* xhat, float a,
                                            float xx, int lane) {
  constexpr int E = (D + 31) / 32;
  float dot = 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane + 32 * e;
    if (d < D) dot = fmaf(xhat[d], g[e], dot);
  }
  dot = warp_sum32(dot);
  const bool proj = sqrtf(xx) > 1e-12f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane + 32 * e;
    if (d < D) g[e] = a * (proj ? g[e] - xhat[d] * dot : g[e]);
  }
}

// Where row pos of head h sits in pattern (w, r): its index in the sparsified
// segment (-1 when the pattern does not keep it), the segment's first kept
// position and its number of kept rows (the last segment ends with the
// sequence).
struct Kept {
  int64_t idx, first, m;
};
__device__ __forceinline__ Kept kept_in(int64_t pos, int64_t h, int64_t w, int64_t r,
                                        int64_t N) {
  Kept k;
  const int64_t seg_start = (pos / w) * w;
  const int64_t o = h % r;
  const int64_t off = pos - seg_start - o;
  k.first = seg_start + o;
  const int64_t len = N - seg_start < w ? N - seg_start : w;
  k.m = len > o ? (len - o + r - 1) / r : 0;
  k.idx = (off < 0 || off % r != 0) ? -1 : off / r;
  return k;
}

// dq: one warp per query row (b, pos, h).  Lane l scores key l of each block
// of 32 keys; the block's score cotangents are then broadcast so that each
// lane adds up its output dims l, l + 32, ...
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dq_kernel(const Problem p, const BwdArgs g) {
  constexpr int E = (D + 31) / 32;
  __shared__ float qsh[kBwdWarps][D];
  __shared__ float dosh[kBwdWarps][D];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * kBwdWarps + warp;
  if (row >= p.B * p.N * p.H) return;
  const int64_t h = row % p.H;
  const int64_t pos = (row / p.H) % p.N;
  const int64_t b = row / (p.H * p.N);
  const T* Q = static_cast<const T*>(p.q);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const T* O = static_cast<const T*>(g.out);
  const T* dO = static_cast<const T*>(g.dout);
  const int64_t HD = p.H * (int64_t)D;
  const int64_t base_b = b * p.N * HD;
  const int64_t me = base_b + pos * HD + h * D;

  float delta = 0.f, qq = 0.f;
  for (int d = lane; d < D; d += 32) {
    const float xq = ld(Q + me + d);
    qsh[warp][d] = xq;
    qq = fmaf(xq, xq, qq);
    const float x = ld(dO + me + d);
    dosh[warp][d] = x;
    delta = fmaf(x, ld(O + me + d), delta);
  }
  delta = warp_sum32(delta);
  qq = warp_sum32(qq);
  __syncwarp();
  // qk_norm: the scores use qhat = a_q q, a_q = 1 / max(|q|, 1e-12)
  const float a_q = p.qk_norm ? 1.f / fmaxf(sqrtf(qq), 1e-12f) : 1.f;
  if (p.qk_norm) {
    for (int d = lane; d < D; d += 32) qsh[warp][d] *= a_q;
    __syncwarp();
  }
  const float lse_i = p.lse[(b * p.H + h) * p.N + pos];
  const float scale = rsqrtf((float)D);
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;

  if (lse_i != -INFINITY) {  // a row no pattern keeps has no gradient
    for (int pi = 0; pi < p.n_pat; ++pi) {
      const int64_t r = p.r[pi];
      const Kept kp = kept_in(pos, h, p.w[pi], r, p.N);
      if (kp.idx < 0) continue;
      const int64_t n_keys = p.causal ? kp.idx + 1 : kp.m;
      for (int64_t j0 = 0; j0 < n_keys; j0 += 32) {
        const int64_t j = j0 + lane;
        float ds = 0.f;
        if (j < n_keys) {
          const int64_t off = base_b + (kp.first + r * j) * HD + h * D;
          float s = 0.f, dp = 0.f, kk = 0.f;
#pragma unroll 16
          for (int d = 0; d < D; ++d) {
            const float xk = ld(K + off + d);
            s = fmaf(qsh[warp][d], xk, s);
            kk = fmaf(xk, xk, kk);
            dp = fmaf(dosh[warp][d], ld(V + off + d), dp);
          }
          // qk_norm: khat = a_k k, so dqhat gets ds * a_k * k
          const float a_k = p.qk_norm ? 1.f / fmaxf(sqrtf(kk), 1e-12f) : 1.f;
          ds = expf(s * a_k * scale - lse_i) * (dp - delta) * a_k;
        }
        const int cnt = (n_keys - j0 < 32) ? (int)(n_keys - j0) : 32;
        for (int t = 0; t < cnt; ++t) {
          const float dst = __shfl_sync(0xffffffffu, ds, t);
          const T* krow = K + base_b + (kp.first + r * (j0 + t)) * HD + h * D;
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int d = lane + 32 * e;
            if (d < D) acc[e] = fmaf(dst, ld(krow + d), acc[e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] *= scale;
  if (p.qk_norm) project_row<D>(acc, qsh[warp], a_q, qq, lane);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane + 32 * e;
    if (d < D) g.dq[me + d] = acc[e];
  }
}

// dk and dv: one warp per key row (b, pos, h).  Lane l takes query l of each
// block of 32 queries (P, delta and the score cotangent); the block is then
// broadcast so that each lane adds up its dims of dk (from q rows) and dv
// (from dout rows).
template <typename T, int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dkv_kernel(const Problem p, const BwdArgs g) {
  constexpr int E = (D + 31) / 32;
  __shared__ float ksh[kBwdWarps][D];
  __shared__ float vsh[kBwdWarps][D];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int64_t row = (int64_t)blockIdx.x * kBwdWarps + warp;
  if (row >= p.B * p.N * p.H) return;
  const int64_t h = row % p.H;
  const int64_t pos = (row / p.H) % p.N;
  const int64_t b = row / (p.H * p.N);
  const T* Q = static_cast<const T*>(p.q);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const T* O = static_cast<const T*>(g.out);
  const T* dO = static_cast<const T*>(g.dout);
  const int64_t HD = p.H * (int64_t)D;
  const int64_t base_b = b * p.N * HD;
  const int64_t me = base_b + pos * HD + h * D;
  const float* lse_bh = p.lse + (b * p.H + h) * p.N;

  float kk = 0.f;
  for (int d = lane; d < D; d += 32) {
    const float xk = ld(K + me + d);
    ksh[warp][d] = xk;
    kk = fmaf(xk, xk, kk);
    vsh[warp][d] = ld(V + me + d);
  }
  kk = warp_sum32(kk);
  __syncwarp();
  // qk_norm: the scores use khat = a_k k
  const float a_k = p.qk_norm ? 1.f / fmaxf(sqrtf(kk), 1e-12f) : 1.f;
  if (p.qk_norm) {
    for (int d = lane; d < D; d += 32) ksh[warp][d] *= a_k;
    __syncwarp();
  }
  const float scale = rsqrtf((float)D);
  float acc_k[E], acc_v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc_k[e] = acc_v[e] = 0.f;

  for (int pi = 0; pi < p.n_pat; ++pi) {
    const int64_t r = p.r[pi];
    const Kept kp = kept_in(pos, h, p.w[pi], r, p.N);
    if (kp.idx < 0) continue;
    const int64_t t0 = p.causal ? kp.idx : 0;
    for (int64_t i0 = t0; i0 < kp.m; i0 += 32) {
      const int64_t i = i0 + lane;
      float pr = 0.f, ds = 0.f;
      if (i < kp.m) {
        const int64_t qpos = kp.first + r * i;
        const int64_t off = base_b + qpos * HD + h * D;
        float s = 0.f, dp = 0.f, delta = 0.f, qq = 0.f;
#pragma unroll 16
        for (int d = 0; d < D; ++d) {
          const float x = ld(dO + off + d);
          const float xq = ld(Q + off + d);
          s = fmaf(xq, ksh[warp][d], s);
          qq = fmaf(xq, xq, qq);
          dp = fmaf(x, vsh[warp][d], dp);
          delta = fmaf(x, ld(O + off + d), delta);
        }
        // qk_norm: qhat = a_q q, so dkhat gets ds * a_q * q
        const float a_q = p.qk_norm ? 1.f / fmaxf(sqrtf(qq), 1e-12f) : 1.f;
        pr = expf(s * a_q * scale - lse_bh[qpos]);
        ds = pr * (dp - delta) * a_q;
      }
      const int cnt = (kp.m - i0 < 32) ? (int)(kp.m - i0) : 32;
      for (int t = 0; t < cnt; ++t) {
        const float pt = __shfl_sync(0xffffffffu, pr, t);
        const float dst = __shfl_sync(0xffffffffu, ds, t);
        const int64_t off = base_b + (kp.first + r * (i0 + t)) * HD + h * D;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int d = lane + 32 * e;
          if (d < D) {
            acc_v[e] = fmaf(pt, ld(dO + off + d), acc_v[e]);
            acc_k[e] = fmaf(dst, ld(Q + off + d), acc_k[e]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) acc_k[e] *= scale;
  if (p.qk_norm) project_row<D>(acc_k, ksh[warp], a_k, kk, lane);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane + 32 * e;
    if (d < D) {
      g.dk[me + d] = acc_k[e];
      g.dv[me + d] = acc_v[e];
    }
  }
}

// ---------------------------------------------------------------- SIMT launch

template <typename T, int D>
int launch_simt_bwd_d(const Problem& p, const BwdArgs& g, dim3 grid, cudaStream_t stream) {
  bwd_dq_kernel<T, D><<<grid, kBwdWarps * 32, 0, stream>>>(p, g);
  if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  bwd_dkv_kernel<T, D><<<grid, kBwdWarps * 32, 0, stream>>>(p, g);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

template <typename T>
int launch_simt_bwd_typed(const Problem& p, const BwdArgs& g, cudaStream_t stream) {
  const int64_t blocks = (p.B * p.N * p.H + kBwdWarps - 1) / kBwdWarps;
  if (blocks > 0x7fffffffLL) return LONGNET_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)blocks);
  switch (p.D) {
    case 16: return launch_simt_bwd_d<T, 16>(p, g, grid, stream);
    case 32: return launch_simt_bwd_d<T, 32>(p, g, grid, stream);
    case 64: return launch_simt_bwd_d<T, 64>(p, g, grid, stream);
    case 128: return launch_simt_bwd_d<T, 128>(p, g, grid, stream);
    default: return LONGNET_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------- tile family

constexpr int kFmtF16 = 0, kFmtBF16 = 1;
constexpr int kTile = 64;            // rows per tile
constexpr int kTileBytes = 64 * 128;  // 64 rows x 64 dims x 2 bytes
constexpr float kLog2e = 1.4426950408889634f;

struct TileParams {
  Problem pb;
  BwdArgs g;
  int64_t unit_base[LONGNET_MAX_PATTERNS + 1];  // prefix sums of B * H * n_seg[p]
  int64_t n_seg[LONGNET_MAX_PATTERNS];
  float scale;       // 1 / sqrt(D)
  float scale_log2;  // log2(e) / sqrt(D)
};

// One sparsified segment: kept row t sits at position first + r * t, t < m.
struct SegRef {
  int64_t b, h, first, r, m;
};

__device__ __forceinline__ SegRef decode_unit(const TileParams& P, int64_t x) {
  int p = 0;
  while (p + 1 < P.pb.n_pat && x >= P.unit_base[p + 1]) ++p;
  int64_t rem = x - P.unit_base[p];
  const int64_t ns = P.n_seg[p];
  const int64_t seg = rem % ns;
  rem /= ns;
  SegRef s;
  s.h = rem % P.pb.H;
  s.b = rem / P.pb.H;
  const int64_t w = P.pb.w[p];
  s.r = P.pb.r[p];
  const int64_t o = s.h % s.r;
  const int64_t len = P.pb.N - seg * w < w ? P.pb.N - seg * w : w;
  s.m = len > o ? (len - o + s.r - 1) / s.r : 0;
  s.first = seg * w + o;
  return s;
}

__device__ __forceinline__ int64_t row_elem(const TileParams& P, const SegRef& s, int64_t t) {
  return ((s.b * P.pb.N + s.first + s.r * t) * P.pb.H + s.h) * 64;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int kPending>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kPending) : "memory");
}

// Byte address of 16-byte chunk ch of row `row` in a tile of 128-byte rows,
// the chunk index XOR-ed with the row's low 3 bits (conflict-free ldmatrix).
__device__ __forceinline__ uint32_t tile_addr(uint32_t base, int row, int ch) {
  return base + (uint32_t)row * 128u + ((uint32_t)(ch ^ (row & 7)) << 4);
}

// Rows t0 .. t0 + 63 of X (16-bit elements) into a tile; rows at or past m
// are zero-filled (no bytes read).  128 threads, 4 chunks each.
__device__ __forceinline__ void load_tile(uint32_t dst, const uint16_t* X, const TileParams& P,
                                          const SegRef& s, int64_t t0, int tid) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int c = tid + 128 * i;
    const int row = c >> 3, ch = c & 7;
    const bool ok = t0 + row < s.m;
    const uint16_t* src = X + row_elem(P, s, ok ? t0 + row : 0) + ch * 8;
    cp_async16(tile_addr(dst, row, ch), src, ok);
  }
}

// lse of rows t0 .. t0 + 63 (zero past m) into 64 floats.
__device__ __forceinline__ void load_lse(uint32_t dst, const TileParams& P, const SegRef& s,
                                         int64_t t0, int tid) {
  if (tid < kTile) {
    const bool ok = t0 + tid < s.m;
    const float* src =
        P.pb.lse + (s.b * P.pb.H + s.h) * P.pb.N + s.first + s.r * (ok ? t0 + tid : 0);
    cp_async4(dst + 4u * tid, src, ok);
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D += A * B, m16n8k16, 16-bit operands of one format, fp32 accumulators.
template <int kFmt>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (kFmt == kFmtBF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}
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

// Per 64-row tile of rows (t0 ..): delta_t = <dout_t, out_t> from two
// swizzled tiles, and lse in place turned to the log2 domain.  Thread pairs
// share a row (32 dims each).
template <int kFmt>
__device__ __forceinline__ void tile_delta(uint32_t s_do, uint32_t s_o, float* lse, float* delta,
                                           int tid) {
  const int row = tid >> 1, half = tid & 1;
  float d = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int ch = 4 * half + c;
    uint32_t a[4], o[4];
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
                 : "r"(tile_addr(s_do, row, ch)));
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3])
                 : "r"(tile_addr(s_o, row, ch)));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x0, x1, y0, y1;
      unpack2<kFmt>(a[e], x0, x1);
      unpack2<kFmt>(o[e], y0, y1);
      d = fmaf(x0, y0, d);
      d = fmaf(x1, y1, d);
    }
  }
  d += __shfl_xor_sync(0xffffffffu, d, 1);
  if (half == 0) {
    delta[row] = d;
    lse[row] *= kLog2e;
  }
}

// qk_norm: the 64 rows of a swizzled tile scaled in place to xhat = a x,
// a = 1 / max(|x|, 1e-12) (rounded back to the 16-bit format, so every
// product sees |xhat| <= 1), and a of each row into a[].  Thread pairs share
// a row; no thread touches another pair's row.
constexpr float kInvNormEps = 1e12f;  // 1 / 1e-12: a row with |x| <= 1e-12 has this a
template <int kFmt>
__device__ __forceinline__ void tile_normalize(uint32_t s_x, float* a, int tid) {
  const int row = tid >> 1, half = tid & 1;
  uint32_t x[4][4];
  float n = 0.f;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(x[c][0]), "=r"(x[c][1]), "=r"(x[c][2]), "=r"(x[c][3])
                 : "r"(tile_addr(s_x, row, 4 * half + c)));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x0, x1;
      unpack2<kFmt>(x[c][e], x0, x1);
      n = fmaf(x0, x0, n);
      n = fmaf(x1, x1, n);
    }
  }
  n += __shfl_xor_sync(0xffffffffu, n, 1);
  const float ar = 1.f / fmaxf(sqrtf(n), 1e-12f);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t y[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x0, x1;
      unpack2<kFmt>(x[c][e], x0, x1);
      y[e] = pack2<kFmt>(x0 * ar, x1 * ar);
    }
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(tile_addr(s_x, row, 4 * half + c)),
                 "r"(y[0]), "r"(y[1]), "r"(y[2]), "r"(y[3])
                 : "memory");
  }
  if (half == 0) a[row] = ar;
}

// qk_norm, at the end of a tile kernel: this lane's gradient g[nt][2 half ..]
// of xhat (rows row0 + 8 half of the normalised tile in s_x, dims
// nt * 8 + 2 t4 + {0, 1}) turned into the gradient of x:
// a (g - xhat <xhat, g>), or a g for a row with |x| <= 1e-12.  The four lanes
// of a row add up <xhat, g>.
template <int kFmt>
__device__ __forceinline__ void tile_project(float (&gr)[8][4], uint32_t s_x, int row0, int t4,
                                             const float (&a)[2]) {
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float xh[8][2];
    float dot = 0.f;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      uint32_t u;
      asm volatile("ld.shared.u32 %0, [%1];"
                   : "=r"(u)
                   : "r"(tile_addr(s_x, row0 + 8 * half, nt) + 4u * t4));
      unpack2<kFmt>(u, xh[nt][0], xh[nt][1]);
      dot = fmaf(xh[nt][0], gr[nt][2 * half], dot);
      dot = fmaf(xh[nt][1], gr[nt][2 * half + 1], dot);
    }
    dot += __shfl_xor_sync(0xffffffffu, dot, 1);
    dot += __shfl_xor_sync(0xffffffffu, dot, 2);
    const bool proj = a[half] < kInvNormEps;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float v = gr[nt][2 * half + e];
        gr[nt][2 * half + e] = a[half] * (proj ? v - xh[nt][e] * dot : v);
      }
    }
  }
}

// Shared memory of the dk/dv kernel (bytes from a 1024-aligned base): K and V
// tiles, then two stages of (Q, dout, out) tiles, two stages of lse, delta.
constexpr int kKvK = 0, kKvV = kTileBytes, kKvStage = 2 * kTileBytes;
constexpr int kKvStageBytes = 3 * kTileBytes;
constexpr int kKvLse = kKvStage + 2 * kKvStageBytes;
constexpr int kKvDelta = kKvLse + 2 * 256;
constexpr int kKvNormK = kKvDelta + 256;  // qk_norm: a of the key rows
constexpr int kKvNormQ = kKvNormK + 256;  // qk_norm: a of the current query rows
constexpr int kKvSmem = kKvNormQ + 256 + 1024;

// dk, dv: CTA (unit = blockIdx.x, key tile jt = blockIdx.y); four warps, warp
// w owns key rows 16 w .. 16 w + 15 of the tile.
template <int kFmt, bool kNorm>
__global__ void __launch_bounds__(128, 3) bwd_dkv_tile_kernel(const __grid_constant__ TileParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const SegRef s = decode_unit(P, blockIdx.x);
  const int64_t T = (s.m + kTile - 1) / kTile;
  const int64_t jt = blockIdx.y;
  if (jt >= T) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const uint32_t sb = smem_u32(smem);
  float* sLse = reinterpret_cast<float*>(smem + kKvLse);
  float* sDelta = reinterpret_cast<float*>(smem + kKvDelta);
  float* sAk = reinterpret_cast<float*>(smem + kKvNormK);
  float* sAq = reinterpret_cast<float*>(smem + kKvNormQ);
  float aK[2] = {1.f, 1.f};  // qk_norm: a of this lane's key rows
  (void)sAk;  // sAk, sAq: the qk_norm instantiation only
  (void)sAq;
  const uint16_t* Q = static_cast<const uint16_t*>(P.pb.q);
  const uint16_t* K = static_cast<const uint16_t*>(P.pb.k);
  const uint16_t* V = static_cast<const uint16_t*>(P.pb.v);
  const uint16_t* O = static_cast<const uint16_t*>(P.g.out);
  const uint16_t* dO = static_cast<const uint16_t*>(P.g.dout);
  const bool causal = P.pb.causal != 0;

  load_tile(sb + kKvK, K, P, s, jt * kTile, tid);
  load_tile(sb + kKvV, V, P, s, jt * kTile, tid);
  const int64_t it0 = causal ? jt : 0;
  {
    const uint32_t st0 = sb + kKvStage;
    load_tile(st0, Q, P, s, it0 * kTile, tid);
    load_tile(st0 + kTileBytes, dO, P, s, it0 * kTile, tid);
    load_tile(st0 + 2 * kTileBytes, O, P, s, it0 * kTile, tid);
    load_lse(sb + kKvLse, P, s, it0 * kTile, tid);
  }
  cp_async_commit();

  float dk[8][4], dv[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[nt][e] = dv[nt][e] = 0.f;
  const int64_t kr0 = jt * kTile + 16 * warp + g;  // this lane's key rows kr0, kr0 + 8
  const uint32_t k_row = sb + kKvK, v_row = sb + kKvV;

  for (int64_t it = it0; it < T; ++it) {
    const int stage = (int)((it - it0) & 1);
    if (it + 1 < T) {
      const uint32_t nx = sb + kKvStage + (stage ^ 1) * kKvStageBytes;
      load_tile(nx, Q, P, s, (it + 1) * kTile, tid);
      load_tile(nx + kTileBytes, dO, P, s, (it + 1) * kTile, tid);
      load_tile(nx + 2 * kTileBytes, O, P, s, (it + 1) * kTile, tid);
      load_lse(sb + kKvLse + (stage ^ 1) * 256, P, s, (it + 1) * kTile, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sQ = sb + kKvStage + stage * kKvStageBytes;
    const uint32_t sdO = sQ + kTileBytes;
    float* lse = sLse + stage * 64;
    tile_delta<kFmt>(sdO, sQ + 2 * kTileBytes, lse, sDelta, tid);
    if constexpr (kNorm) {  // q rows, and once the key rows, to unit norm
      tile_normalize<kFmt>(sQ, sAq, tid);
      if (it == it0) tile_normalize<kFmt>(k_row, sAk, tid);
    }
    __syncthreads();
    if constexpr (kNorm) {
      if (it == it0) {
        aK[0] = sAk[16 * warp + g];
        aK[1] = sAk[16 * warp + g + 8];
      }
    }

#pragma unroll
    for (int hq = 0; hq < 2; ++hq) {  // 32 queries at a time
      float st[4][4], dpt[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[nt][e] = dpt[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {  // 16 dims per step
        uint32_t ak[4], av[4];
        ldsm_x4(tile_addr(k_row, 16 * warp + (lane & 15), 2 * kk + (lane >> 4)), ak);
        ldsm_x4(tile_addr(v_row, 16 * warp + (lane & 15), 2 * kk + (lane >> 4)), av);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          const int qr = (2 * hq + np) * 16 + (lane & 7) + ((lane >> 4) << 3);
          uint32_t bq[4], bd[4];
          ldsm_x4(tile_addr(sQ, qr, 2 * kk + ((lane >> 3) & 1)), bq);
          ldsm_x4(tile_addr(sdO, qr, 2 * kk + ((lane >> 3) & 1)), bd);
          mma16816<kFmt>(st[2 * np], ak, bq[0], bq[1]);
          mma16816<kFmt>(st[2 * np + 1], ak, bq[2], bq[3]);
          mma16816<kFmt>(dpt[2 * np], av, bd[0], bd[1]);
          mma16816<kFmt>(dpt[2 * np + 1], av, bd[2], bd[3]);
        }
      }
      // P^T and dS^T for rows (keys) kr0, kr0 + 8 and this lane's query columns
      uint32_t pa[2][4], da[2][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float pv[4], dsv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int qc = 32 * hq + nt * 8 + 2 * t4 + (e & 1);
          const int64_t qi = it * kTile + qc;
          const int64_t kr = kr0 + ((e >> 1) << 3);
          const bool ok = qi < s.m && kr < s.m && (!causal || qi >= kr);
          const float pr = ok ? ex2(fmaf(st[nt][e], P.scale_log2, -lse[qc])) : 0.f;
          pv[e] = pr;
          dsv[e] = pr * (dpt[nt][e] - sDelta[qc]);
        }
        const int kq = nt >> 1, hi = nt & 1;
        pa[kq][2 * hi] = pack2<kFmt>(pv[0], pv[1]);
        pa[kq][2 * hi + 1] = pack2<kFmt>(pv[2], pv[3]);
        da[kq][2 * hi] = pack2<kFmt>(dsv[0], dsv[1]);
        da[kq][2 * hi + 1] = pack2<kFmt>(dsv[2], dsv[3]);
      }
      // dV += P^T dout, dK += dS^T q over these 32 queries
#pragma unroll
      for (int kq = 0; kq < 2; ++kq) {
        const int qr = (2 * hq + kq) * 16 + (lane & 15);
#pragma unroll
        for (int dp = 0; dp < 4; ++dp) {
          uint32_t bd[4], bq[4];
          ldsm_x4_t(tile_addr(sdO, qr, 2 * dp + (lane >> 4)), bd);
          ldsm_x4_t(tile_addr(sQ, qr, 2 * dp + (lane >> 4)), bq);
          mma16816<kFmt>(dv[2 * dp], pa[kq], bd[0], bd[1]);
          mma16816<kFmt>(dv[2 * dp + 1], pa[kq], bd[2], bd[3]);
          mma16816<kFmt>(dk[2 * dp], da[kq], bq[0], bq[1]);
          mma16816<kFmt>(dk[2 * dp + 1], da[kq], bq[2], bq[3]);
        }
      }
    }
    __syncthreads();  // the stage is refilled two iterations on
  }
  cp_async_wait<0>();
  if constexpr (kNorm) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dk[nt][e] *= P.scale;
    tile_project<kFmt>(dk, k_row, 16 * warp + g, t4, aK);
  }
  const float dk_scale = kNorm ? 1.f : P.scale;

  // one fp32 add per pattern into the caller's gradients
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int64_t kr = kr0 + 8 * half;
    if (kr < s.m) {
      const int64_t off = row_elem(P, s, kr);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int d = nt * 8 + 2 * t4;
        atomicAdd(reinterpret_cast<float2*>(P.g.dk + off + d),
                  make_float2(dk[nt][2 * half] * dk_scale, dk[nt][2 * half + 1] * dk_scale));
        atomicAdd(reinterpret_cast<float2*>(P.g.dv + off + d),
                  make_float2(dv[nt][2 * half], dv[nt][2 * half + 1]));
      }
    }
  }
}

// Shared memory of the dq kernel: Q, dout, out tiles of the CTA's query tile,
// two stages of (K, V) tiles, lse, delta.
constexpr int kQQ = 0, kQdO = kTileBytes, kQO = 2 * kTileBytes, kQStage = 3 * kTileBytes;
constexpr int kQStageBytes = 2 * kTileBytes;
constexpr int kQLse = kQStage + 2 * kQStageBytes;
constexpr int kQDelta = kQLse + 256;
constexpr int kQNormQ = kQDelta + 256;  // qk_norm: a of the query rows
constexpr int kQNormK = kQNormQ + 256;  // qk_norm: a of the current key rows
constexpr int kQSmem = kQNormK + 256 + 1024;

// dq: CTA (unit = blockIdx.x, query tile it = T - 1 - blockIdx.y, the
// costliest first when causal); warp w owns query rows 16 w .. 16 w + 15.
template <int kFmt, bool kNorm>
__global__ void __launch_bounds__(128) bwd_dq_tile_kernel(const __grid_constant__ TileParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const SegRef s = decode_unit(P, blockIdx.x);
  const int64_t T = (s.m + kTile - 1) / kTile;
  if ((int64_t)blockIdx.y >= T) return;
  const int64_t it = T - 1 - blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  const uint32_t sb = smem_u32(smem);
  float* sLse = reinterpret_cast<float*>(smem + kQLse);
  float* sDelta = reinterpret_cast<float*>(smem + kQDelta);
  float* sAq = reinterpret_cast<float*>(smem + kQNormQ);
  float* sAk = reinterpret_cast<float*>(smem + kQNormK);
  float aQ[2] = {1.f, 1.f};  // qk_norm: a of this lane's query rows
  (void)sAq;  // sAq, sAk: the qk_norm instantiation only
  (void)sAk;
  const uint16_t* Q = static_cast<const uint16_t*>(P.pb.q);
  const uint16_t* K = static_cast<const uint16_t*>(P.pb.k);
  const uint16_t* V = static_cast<const uint16_t*>(P.pb.v);
  const uint16_t* O = static_cast<const uint16_t*>(P.g.out);
  const uint16_t* dO = static_cast<const uint16_t*>(P.g.dout);
  const bool causal = P.pb.causal != 0;

  load_tile(sb + kQQ, Q, P, s, it * kTile, tid);
  load_tile(sb + kQdO, dO, P, s, it * kTile, tid);
  load_tile(sb + kQO, O, P, s, it * kTile, tid);
  load_lse(sb + kQLse, P, s, it * kTile, tid);
  load_tile(sb + kQStage, K, P, s, 0, tid);
  load_tile(sb + kQStage + kTileBytes, V, P, s, 0, tid);
  cp_async_commit();

  float dq[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;
  const int64_t qr0 = it * kTile + 16 * warp + g;  // this lane's query rows qr0, qr0 + 8
  const int64_t jt_end = causal ? it + 1 : T;
  float lse2[2] = {0.f, 0.f}, dlt[2] = {0.f, 0.f};

  for (int64_t jt = 0; jt < jt_end; ++jt) {
    const int stage = (int)(jt & 1);
    if (jt + 1 < jt_end) {
      const uint32_t nx = sb + kQStage + (stage ^ 1) * kQStageBytes;
      load_tile(nx, K, P, s, (jt + 1) * kTile, tid);
      load_tile(nx + kTileBytes, V, P, s, (jt + 1) * kTile, tid);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const uint32_t sK = sb + kQStage + stage * kQStageBytes;
    if (jt == 0) {
      tile_delta<kFmt>(sb + kQdO, sb + kQO, sLse, sDelta, tid);
      if constexpr (kNorm) tile_normalize<kFmt>(sb + kQQ, sAq, tid);
      __syncthreads();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        lse2[half] = sLse[16 * warp + g + 8 * half];
        dlt[half] = sDelta[16 * warp + g + 8 * half];
        if constexpr (kNorm) aQ[half] = sAq[16 * warp + g + 8 * half];
      }
    }
    if constexpr (kNorm) {  // the key rows to unit norm
      tile_normalize<kFmt>(sK, sAk, tid);
      __syncthreads();
    }
    const uint32_t sV = sK + kTileBytes;
#pragma unroll
    for (int hk = 0; hk < 2; ++hk) {  // 32 keys at a time
      float sc[4][4], dp[4][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sc[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t aq[4], ad[4];
        ldsm_x4(tile_addr(sb + kQQ, 16 * warp + (lane & 15), 2 * kk + (lane >> 4)), aq);
        ldsm_x4(tile_addr(sb + kQdO, 16 * warp + (lane & 15), 2 * kk + (lane >> 4)), ad);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          const int kr = (2 * hk + np) * 16 + (lane & 7) + ((lane >> 4) << 3);
          uint32_t bk[4], bv[4];
          ldsm_x4(tile_addr(sK, kr, 2 * kk + ((lane >> 3) & 1)), bk);
          ldsm_x4(tile_addr(sV, kr, 2 * kk + ((lane >> 3) & 1)), bv);
          mma16816<kFmt>(sc[2 * np], aq, bk[0], bk[1]);
          mma16816<kFmt>(sc[2 * np + 1], aq, bk[2], bk[3]);
          mma16816<kFmt>(dp[2 * np], ad, bv[0], bv[1]);
          mma16816<kFmt>(dp[2 * np + 1], ad, bv[2], bv[3]);
        }
      }
      uint32_t da[2][4];
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
        float dsv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t kj = jt * kTile + 32 * hk + nt * 8 + 2 * t4 + (e & 1);
          const int64_t qi = qr0 + ((e >> 1) << 3);
          const bool ok = kj < s.m && (!causal || kj <= qi);
          const float pr = ok ? ex2(fmaf(sc[nt][e], P.scale_log2, -lse2[e >> 1])) : 0.f;
          dsv[e] = pr * (dp[nt][e] - dlt[e >> 1]);
        }
        const int kq = nt >> 1, hi = nt & 1;
        da[kq][2 * hi] = pack2<kFmt>(dsv[0], dsv[1]);
        da[kq][2 * hi + 1] = pack2<kFmt>(dsv[2], dsv[3]);
      }
      // dQ += dS K over these 32 keys
#pragma unroll
      for (int kq = 0; kq < 2; ++kq) {
        const int kr = (2 * hk + kq) * 16 + (lane & 15);
#pragma unroll
        for (int dd = 0; dd < 4; ++dd) {
          uint32_t bk[4];
          ldsm_x4_t(tile_addr(sK, kr, 2 * dd + (lane >> 4)), bk);
          mma16816<kFmt>(dq[2 * dd], da[kq], bk[0], bk[1]);
          mma16816<kFmt>(dq[2 * dd + 1], da[kq], bk[2], bk[3]);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  if constexpr (kNorm) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dq[nt][e] *= P.scale;
    tile_project<kFmt>(dq, sb + kQQ, 16 * warp + g, t4, aQ);
  }
  const float dq_scale = kNorm ? 1.f : P.scale;

#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int64_t qi = qr0 + 8 * half;
    if (qi < s.m) {
      const int64_t off = row_elem(P, s, qi);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int d = nt * 8 + 2 * t4;
        atomicAdd(reinterpret_cast<float2*>(P.g.dq + off + d),
                  make_float2(dq[nt][2 * half] * dq_scale, dq[nt][2 * half + 1] * dq_scale));
      }
    }
  }
}

// Units and the tile count of the tallest segment; false when the grid would
// not fit (then the SIMT family takes the call).
bool tile_geometry(const Problem& p, TileParams* tp, int64_t* t_max) {
  int64_t units = 0, tm = 0;
  for (int i = 0; i < p.n_pat; ++i) {
    const int64_t n_seg = (p.N + p.w[i] - 1) / p.w[i];
    const int64_t wl = p.w[i] < p.N ? p.w[i] : p.N;
    const int64_t m_max = (wl + p.r[i] - 1) / p.r[i];  // o = 0 keeps the most rows
    const int64_t t = (m_max + kTile - 1) / kTile;
    if (t > tm) tm = t;
    if (tp) {
      tp->unit_base[i] = units;
      tp->n_seg[i] = n_seg;
    }
    units += p.B * p.H * n_seg;
  }
  if (tp) tp->unit_base[p.n_pat] = units;
  *t_max = tm;
  return units > 0 && units <= 0x7fffffffLL && tm >= 1 && tm <= 65535;
}

template <int kFmt, bool kNorm>
int launch_tile_bwd_fmt(const TileParams& tp, int64_t units, int64_t t_max, cudaStream_t stream) {
  // per device: the attribute is set once on each (setting it twice, from two
  // threads at once, is harmless)
  static std::atomic<bool> attr_set[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  if (!attr_set[dev].load(std::memory_order_acquire)) {
    if (cudaFuncSetAttribute(bwd_dkv_tile_kernel<kFmt, kNorm>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kKvSmem) != cudaSuccess ||
        cudaFuncSetAttribute(bwd_dq_tile_kernel<kFmt, kNorm>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmem) != cudaSuccess) {
      cudaGetLastError();
      return LONGNET_ERR_CUDA;
    }
    attr_set[dev].store(true, std::memory_order_release);
  }
  const dim3 grid((unsigned)units, (unsigned)t_max);
  bwd_dq_tile_kernel<kFmt, kNorm><<<grid, 128, kQSmem, stream>>>(tp);
  if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  bwd_dkv_tile_kernel<kFmt, kNorm><<<grid, 128, kKvSmem, stream>>>(tp);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

int launch_tile_bwd(const Problem& p, const BwdArgs& g, cudaStream_t stream) {
  TileParams tp;
  int64_t t_max = 0;
  if (!tile_geometry(p, &tp, &t_max)) return LONGNET_ERR_UNSUPPORTED;
  tp.pb = p;
  tp.g = g;
  tp.scale = 1.f / sqrtf((float)p.D);
  tp.scale_log2 = kLog2e * tp.scale;
  const size_t bytes = sizeof(float) * (size_t)(p.B * p.N * p.H * p.D);
  if (cudaMemsetAsync(g.dq, 0, bytes, stream) != cudaSuccess ||
      cudaMemsetAsync(g.dk, 0, bytes, stream) != cudaSuccess ||
      cudaMemsetAsync(g.dv, 0, bytes, stream) != cudaSuccess) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  const int64_t units = tp.unit_base[p.n_pat];
  if (p.qk_norm) {
    if (p.dtype == LONGNET_DTYPE_F16) return launch_tile_bwd_fmt<kFmtF16, true>(tp, units, t_max, stream);
    return launch_tile_bwd_fmt<kFmtBF16, true>(tp, units, t_max, stream);
  }
  if (p.dtype == LONGNET_DTYPE_F16) return launch_tile_bwd_fmt<kFmtF16, false>(tp, units, t_max, stream);
  return launch_tile_bwd_fmt<kFmtBF16, false>(tp, units, t_max, stream);
}

}  // namespace

bool backward_supports(const Problem& p) {
  return p.D == 16 || p.D == 32 || p.D == 64 || p.D == 128;
}

bool tile_backward_supports(const Problem& p) {
  int64_t t_max = 0;
  return p.D == 64 &&
         (p.dtype == LONGNET_DTYPE_BF16 || p.dtype == LONGNET_DTYPE_F16) &&
         tile_geometry(p, nullptr, &t_max);
}

int launch_backward(const Problem& p, const BwdArgs& g, int impl, cudaStream_t stream) {
  if (impl == LONGNET_IMPL_AUTO)
    impl = tcgen05_backward_supports(p) ? LONGNET_IMPL_TCGEN05
                                        : tile_backward_supports(p) ? LONGNET_IMPL_TILES : LONGNET_IMPL_SIMT;
  if (impl == LONGNET_IMPL_TCGEN05) return launch_tcgen05_backward(p, g, stream);
  if (impl == LONGNET_IMPL_TILES) {
    if (!tile_backward_supports(p)) return LONGNET_ERR_UNSUPPORTED;
    return launch_tile_bwd(p, g, stream);
  }
  if (impl != LONGNET_IMPL_SIMT) return LONGNET_ERR_INVALID_ARG;
  if (!backward_supports(p)) return LONGNET_ERR_UNSUPPORTED;
  if (p.dtype == LONGNET_DTYPE_F32) return launch_simt_bwd_typed<float>(p, g, stream);
  if (p.dtype == LONGNET_DTYPE_F16) return launch_simt_bwd_typed<__half>(p, g, stream);
  return launch_simt_bwd_typed<__nv_bfloat16>(p, g, stream);
}

}  // namespace longnet
