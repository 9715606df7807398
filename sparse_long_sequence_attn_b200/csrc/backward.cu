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
// Two fp32 SIMT kernels, one warp per row, neither writing anything but its
// own output rows (no scratch, no atomics):
//   - dq: the row as a query, over the keys of every pattern keeping it (the
//     forward SIMT kernel's walk), recomputing P from q, k and the saved lse;
//   - dk, dv: the row as a key, over the queries of every pattern keeping it
//     (the ones at or after it when causal), recomputing P and delta_i from
//     q, dout, out and lse of each query.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "device_util.cuh"
#include "params.h"

namespace longnet {
namespace {

constexpr int kBwdWarps = 4;

__device__ __forceinline__ float ld(const float* p) { return *p; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld(const __half* p) { return __half2float(*p); }
__device__ __forceinline__ void st(float* p, float x) { *p = x; }
__device__ __forceinline__ void st(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void st(__half* p, float x) { *p = __float2half_rn(x); }

__device__ __forceinline__ float warp_sum32(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
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

  float delta = 0.f;
  for (int d = lane; d < D; d += 32) {
    qsh[warp][d] = ld(Q + me + d);
    const float x = ld(dO + me + d);
    dosh[warp][d] = x;
    delta = fmaf(x, ld(O + me + d), delta);
  }
  delta = warp_sum32(delta);
  __syncwarp();
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
          float s = 0.f, dp = 0.f;
#pragma unroll 16
          for (int d = 0; d < D; ++d) {
            s = fmaf(qsh[warp][d], ld(K + off + d), s);
            dp = fmaf(dosh[warp][d], ld(V + off + d), dp);
          }
          ds = expf(s * scale - lse_i) * (dp - delta);
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
  T* dQ = static_cast<T*>(g.dq);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane + 32 * e;
    if (d < D) st(dQ + me + d, acc[e] * scale);
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

  for (int d = lane; d < D; d += 32) {
    ksh[warp][d] = ld(K + me + d);
    vsh[warp][d] = ld(V + me + d);
  }
  __syncwarp();
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
        float s = 0.f, dp = 0.f, delta = 0.f;
#pragma unroll 16
        for (int d = 0; d < D; ++d) {
          const float x = ld(dO + off + d);
          s = fmaf(ld(Q + off + d), ksh[warp][d], s);
          dp = fmaf(x, vsh[warp][d], dp);
          delta = fmaf(x, ld(O + off + d), delta);
        }
        pr = expf(s * scale - lse_bh[qpos]);
        ds = pr * (dp - delta);
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
  T* dK = static_cast<T*>(g.dk);
  T* dV = static_cast<T*>(g.dv);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane + 32 * e;
    if (d < D) {
      st(dK + me + d, acc_k[e] * scale);
      st(dV + me + d, acc_v[e]);
    }
  }
}

template <typename T, int D>
int launch_bwd_d(const Problem& p, const BwdArgs& g, dim3 grid, cudaStream_t stream) {
  bwd_dq_kernel<T, D><<<grid, kBwdWarps * 32, 0, stream>>>(p, g);
  if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  bwd_dkv_kernel<T, D><<<grid, kBwdWarps * 32, 0, stream>>>(p, g);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

template <typename T>
int launch_bwd_typed(const Problem& p, const BwdArgs& g, cudaStream_t stream) {
  const int64_t blocks = (p.B * p.N * p.H + kBwdWarps - 1) / kBwdWarps;
  if (blocks > 0x7fffffffLL) return LONGNET_ERR_UNSUPPORTED;
  const dim3 grid((unsigned)blocks);
  switch (p.D) {
    case 16: return launch_bwd_d<T, 16>(p, g, grid, stream);
    case 32: return launch_bwd_d<T, 32>(p, g, grid, stream);
    case 64: return launch_bwd_d<T, 64>(p, g, grid, stream);
    case 128: return launch_bwd_d<T, 128>(p, g, grid, stream);
    default: return LONGNET_ERR_UNSUPPORTED;
  }
}

}  // namespace

bool backward_supports(const Problem& p) {
  return !p.qk_norm && (p.D == 16 || p.D == 32 || p.D == 64 || p.D == 128);
}

int launch_backward(const Problem& p, const BwdArgs& g, cudaStream_t stream) {
  if (p.dtype == LONGNET_DTYPE_F32) return launch_bwd_typed<float>(p, g, stream);
  if (p.dtype == LONGNET_DTYPE_F16) return launch_bwd_typed<__half>(p, g, stream);
  return launch_bwd_typed<__nv_bfloat16>(p, g, stream);
}

}  // namespace longnet
