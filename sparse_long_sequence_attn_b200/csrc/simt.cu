// Kernel family SIMT: fp32 FMA arithmetic, one warp per output row.
//
// The general path of the library (any supported D, fp32 or bf16 inputs, any
// pattern set).  It is also the only path for fp32, because tensor-core TF32
// would not keep fp32 accuracy.
//
// Combining the patterns ("LONGNET: Scaling Transformer to 1 billion tokens",
// section "Token expansion reaches 1 billion+": local attention combined into
// global attention) with weights e^{lse_p} is the same as one softmax over all
// (pattern, key) pairs that reach the row: e^{lse_p} O_p = sum_{j in p}
// e^{s_j} v_j.  So each warp runs a single online softmax over the keys of
// every pattern that keeps its row, and the combination needs no separate
// step.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "device_util.cuh"
#include "params.h"

namespace longnet {
namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ float load_elem(const float* p) { return *p; }
__device__ __forceinline__ float load_elem(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float load_elem(const __half* p) { return __half2float(*p); }
__device__ __forceinline__ void store_elem(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_elem(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }
__device__ __forceinline__ void store_elem(__half* p, float x) { *p = __float2half_rn(x); }

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Dot product of the shared-memory query row with one key row (length D).
template <typename T, int D>
__device__ __forceinline__ float dot_row(const float* qs, const T* krow) {
  float s = 0.f;
#pragma unroll 16
  for (int d = 0; d < D; ++d) s = fmaf(qs[d], load_elem(krow + d), s);
  return s;
}

// The same, also returning the key row's squared norm.
template <typename T, int D>
__device__ __forceinline__ float dot_row_norm(const float* qs, const T* krow, float& kk) {
  float s = 0.f, n = 0.f;
#pragma unroll 16
  for (int d = 0; d < D; ++d) {
    const float x = load_elem(krow + d);
    s = fmaf(qs[d], x, s);
    n = fmaf(x, x, n);
  }
  kk = n;
  return s;
}

// One warp per (b, pos, h).  Lane l owns output dims l, l+32, ... (E of them);
// within a block of 32 keys lane l scores key l, then the block's
// probabilities are broadcast to accumulate V.
template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32) simt_kernel(const Problem p) {
  constexpr int E = (D + 31) / 32;
  __shared__ float qsh[kWarps][D];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  // rows of the computed part: positions [q0, q1), heads [h0, h1)
  const int64_t row = (int64_t)blockIdx.x * kWarps + warp;
  const int64_t Hr = p.h1 - p.h0, Nr = p.q1 - p.q0;
  const int64_t n_rows = p.B * Nr * Hr;
  if (row >= n_rows) return;
  const int64_t h = p.h0 + row % Hr;
  const int64_t pos = p.q0 + (row / Hr) % Nr;
  const int64_t b = row / (Hr * Nr);
  const T* Q = static_cast<const T*>(p.q);
  const T* K = static_cast<const T*>(p.k);
  const T* V = static_cast<const T*>(p.v);
  const int64_t HD = p.H * (int64_t)D;
  const int64_t base_b = b * p.N * HD;

  for (int d = lane; d < D; d += 32) qsh[warp][d] = load_elem(Q + base_b + pos * HD + h * D + d);
  __syncwarp();
  if (p.qk_norm) {
    // q / max(|q|, 1e-12) in fp32; each key row is scaled the same way below
    float ss = 0.f;
    for (int d = lane; d < D; d += 32) ss = fmaf(qsh[warp][d], qsh[warp][d], ss);
    const float inv = 1.f / fmaxf(sqrtf(warp_sum(ss)), 1e-12f);
    __syncwarp();
    for (int d = lane; d < D; d += 32) qsh[warp][d] *= inv;
    __syncwarp();
  }

  const float scale = rsqrtf((float)D);
  float m_run = -INFINITY, l_run = 0.f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;

  for (int pi = 0; pi < p.n_pat; ++pi) {
    const int64_t w = p.w[pi], r = p.r[pi];
    const int64_t seg_start = (pos / w) * w;
    const int64_t o = h % r;
    const int64_t off = pos - seg_start - o;
    if (off < 0 || off % r != 0) continue;  // this pattern does not keep the row
    const int64_t kk = off / r;
    // the last segment ends with the sequence (shorter when w does not divide N)
    const int64_t len = p.N - seg_start < w ? p.N - seg_start : w;
    const int64_t m = (len - o + r - 1) / r;
    const int64_t n_keys = p.causal ? kk + 1 : m;
    const int64_t first = seg_start + o;
    for (int64_t j0 = 0; j0 < n_keys; j0 += 32) {
      const int64_t j = j0 + lane;
      float s = -INFINITY;
      if (j < n_keys) {
        const int64_t kp = first + r * j;
        if (p.qk_norm) {
          float kk;
          s = dot_row_norm<T, D>(qsh[warp], K + base_b + kp * HD + h * D, kk);
          s *= scale / fmaxf(sqrtf(kk), 1e-12f);
        } else {
          s = dot_row<T, D>(qsh[warp], K + base_b + kp * HD + h * D) * scale;
        }
      }
      const float m_new = fmaxf(m_run, warp_max(s));
      const float corr = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
      const float pj = (j < n_keys) ? expf(s - m_new) : 0.f;
      l_run = l_run * corr + warp_sum(pj);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] *= corr;
      const int64_t cnt = (n_keys - j0 < 32) ? (n_keys - j0) : 32;
      for (int t = 0; t < (int)cnt; ++t) {
        const float pt = __shfl_sync(0xffffffffu, pj, t);
        const int64_t kp = first + r * (j0 + t);
        const T* vrow = V + base_b + kp * HD + h * D;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int d = lane + 32 * e;
          if (d < D) acc[e] = fmaf(pt, load_elem(vrow + d), acc[e]);
        }
      }
      m_run = m_new;
    }
  }

  T* O = static_cast<T*>(p.out);
  const float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int d = lane + 32 * e;
    if (d < D) store_elem(O + base_b + pos * HD + h * D + d, acc[e] * inv);
  }
  if (p.lse && lane == 0) {
    p.lse[(b * p.H + h) * p.N + pos] = (l_run > 0.f) ? m_run + logf(l_run) : -INFINITY;
  }
}

template <typename T>
int launch_typed(const Problem& p, cudaStream_t stream) {
  const int64_t n_rows = p.B * (p.q1 - p.q0) * (p.h1 - p.h0);
  const int64_t blocks = (n_rows + kWarps - 1) / kWarps;
  if (blocks > 0x7fffffffLL) return LONGNET_ERR_UNSUPPORTED;
  dim3 grid((unsigned)blocks), block(kWarps * 32);
  switch (p.D) {
    case 16: simt_kernel<T, 16><<<grid, block, 0, stream>>>(p); break;
    case 32: simt_kernel<T, 32><<<grid, block, 0, stream>>>(p); break;
    case 64: simt_kernel<T, 64><<<grid, block, 0, stream>>>(p); break;
    case 128: simt_kernel<T, 128><<<grid, block, 0, stream>>>(p); break;
    default: return LONGNET_ERR_UNSUPPORTED;
  }
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

}  // namespace

int launch_simt(const Problem& p, cudaStream_t stream) {
  if (p.dtype == LONGNET_DTYPE_F32) return launch_typed<float>(p, stream);
  if (p.dtype == LONGNET_DTYPE_F16) return launch_typed<__half>(p, stream);
  return launch_typed<__nv_bfloat16>(p, stream);
}

}  // namespace longnet
