// The input-side prologue of the forward: the query and key rows transformed
// once, before the attention, into a workspace that the attention kernels
// then read in place of q and k.
//
//  * qk_norm: every q row and every k row scaled to unit L2 norm over D,
//    x / max(|x|, 1e-12), in fp32 (the qk_norm option of the DilatedAttention
//    module, "LongNet" docs page, usage example);
//  * XPOS: the rotary position encoding with exponential scaling that the
//    use_xpos option names ("LongNet论文精读", section "Dilated Attention的核心
//    参数解析").  The pages give no formula; the one taken is the published
//    XPOS definition (Sun et al., "A Length-Extrapolatable Transformer"):
//    for the pair of elements (2i, 2i+1) of a row at position n,
//      theta_i = 10000^(-2i / D),   zeta_i = (2i + 0.4 D) / (1.4 D),
//      s = zeta_i^((n - c) / 512),  c = floor(N / 2),
//      (x0, x1) -> s (x0 cos(n theta_i) - x1 sin(n theta_i),
//                     x1 cos(n theta_i) + x0 sin(n theta_i))
//    for queries and the same with s replaced by 1 / s for keys, so that a
//    score q_m . k_n depends on m - n only (the centring c cancels in it and
//    keeps the scales in range).  When both options are set the norm comes
//    first.
//
// The pass is bound by HBM (read q and k, write them once): each thread
// moves 8 consecutive elements (16 bytes of a 16-bit format) of a few heads'
// rows at one position, a row is D / 8 threads of one warp, the norm is a
// shuffle reduction among them, and the grid is a whole number of waves over
// the SMs.  The XPOS factors of a position serve several heads: the angle
// n theta_i is reduced modulo 2 pi in fp64 (n reaches 2^30) before an fp32
// sincos, the scale is an fp32 exp2 of log2(zeta_i) (n - c) / 512, and the
// key scale its reciprocal.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "device_util.cuh"
#include "params.h"

namespace longnet {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxPairs = 64;  // D <= 128

struct XposTable {
  double theta[kMaxPairs];     // 10000^(-2i / D)
  float log2zeta[kMaxPairs];   // log2((2i + 0.4 D) / (1.4 D))
};

__device__ __forceinline__ void load8(const float* p, float* x) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}
__device__ __forceinline__ void store8(float* p, const float* x) {
  reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(h[j]);
    x[2 * j] = f.x;
    x[2 * j + 1] = f.y;
  }
}
__device__ __forceinline__ void store8(__nv_bfloat16* p, const float* x) {
  uint4 u;
  __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
  for (int j = 0; j < 4; ++j) h[j] = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}
__device__ __forceinline__ void load8(const __half* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __half22float2(h[j]);
    x[2 * j] = f.x;
    x[2 * j + 1] = f.y;
  }
}
__device__ __forceinline__ void store8(__half* p, const float* x) {
  uint4 u;
  __half2* h = reinterpret_cast<__half2*>(&u);
#pragma unroll
  for (int j = 0; j < 4; ++j) h[j] = __floats2half2_rn(x[2 * j], x[2 * j + 1]);
  *reinterpret_cast<uint4*>(p) = u;
}

// One thread group of TPR = D / 8 threads (2, 4, 8 or 16) per position
// (b, n) and group of kHG heads: each thread owns 8 consecutive elements
// (4 element pairs) of the group's q rows and k rows at that position.  The
// XPOS factors depend on the position and the pair only, so a thread
// evaluates them once for its 4 pairs and applies them to the 2 kHG rows it
// moves, whose loads are all issued before the first is used.
constexpr int kHG = 4;

template <typename T, int TPR>
__global__ void __launch_bounds__(kThreads)
    prologue_kernel(const T* __restrict__ q, const T* __restrict__ k, T* __restrict__ qo,
                    T* __restrict__ ko, int64_t positions, int N, int H, int center, int qk_norm, int xpos,
                    const XposTable tab) {
  constexpr int kD = TPR * 8;
  const int lane = threadIdx.x & 31;
  const int n_groups = (H + kHG - 1) / kHG;
  const int64_t total = positions * n_groups * TPR;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t base = ((int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5)) * 32; base < total;
       base += warps * 32) {
    // whole warps stay in the loop so the row reductions can shuffle; the TPR
    // threads of a row are either all in range or all out (total is a
    // multiple of TPR)
    const int64_t t = base + lane;
    const bool active = t < total;
    const int chunk = (int)(t % TPR);
    const int64_t u = active ? t / TPR : 0;
    const int h0 = (int)(u % n_groups) * kHG;
    const int64_t pos = u / n_groups;  // b N + n
    float cs[4], sn[4], sc[4];
    if (xpos) {
      const int n = (int)(pos % N);
      const float rel = (float)(n - center) * (1.f / 512.f);
      const double two_pi = 6.283185307179586476925286766559;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = chunk * 4 + j;
        double a = (double)n * tab.theta[i];
        a -= two_pi * rint(a * (1.0 / two_pi));
        sincosf((float)a, &sn[j], &cs[j]);
        sc[j] = exp2f(tab.log2zeta[i] * rel);
      }
    }
    // rows 0 .. kHG-1: q of heads h0 + j; rows kHG .. 2 kHG - 1: k of them
    uint4 raw[2 * kHG][sizeof(T) == 4 ? 2 : 1];
#pragma unroll
    for (int j = 0; j < 2 * kHG; ++j) {
      const int h = h0 + (j % kHG);
      const T* src = (j < kHG ? q : k) + (pos * H + h) * kD + chunk * 8;
#pragma unroll
      for (int c = 0; c < (sizeof(T) == 4 ? 2 : 1); ++c)
        raw[j][c] = (active && h < H) ? reinterpret_cast<const uint4*>(src)[c] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int j = 0; j < 2 * kHG; ++j) {
      const bool is_k = j >= kHG;
      const int h = h0 + (j % kHG);
      float x[8];
      load8(reinterpret_cast<const T*>(&raw[j][0]), x);
      if (qk_norm) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x[e], x[e], ss);
#pragma unroll
        for (int m = 1; m < TPR; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
        const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] *= inv;
      }
      if (xpos) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float s = is_k ? 1.f / sc[e] : sc[e];
          const float x0 = x[2 * e], x1 = x[2 * e + 1];
          x[2 * e] = (x0 * cs[e] - x1 * sn[e]) * s;
          x[2 * e + 1] = (x1 * cs[e] + x0 * sn[e]) * s;
        }
      }
      if (active && h < H) store8((is_k ? ko : qo) + (pos * H + h) * kD + chunk * 8, x);
    }
  }
}

// The backward of the pass: the fp32 gradient g of the encoded rows (in
// place, [B, N, H, D]) becomes the gradient of the original rows x: first
// back through XPOS (per pair the transpose of s R(n theta_i): s R(-n theta_i),
// 1/s for keys), then through the norm, a (g - xhat <xhat, g>) with
// a = 1 / max(|x|, 1e-12) and xhat = a x (a g where |x| <= 1e-12).  One
// thread group of TPR = D / 8 threads per row, 8 elements each.
template <typename T, int TPR>
__global__ void __launch_bounds__(kThreads)
    prologue_bwd_kernel(const T* __restrict__ x, float* __restrict__ g, int64_t rows, int N, int H, int center,
                        int qk_norm, int xpos, int is_k, const XposTable tab) {
  constexpr int kD = TPR * 8;
  const int lane = threadIdx.x & 31;
  const int64_t total = rows * TPR;
  const int64_t warps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t base = ((int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5)) * 32; base < total;
       base += warps * 32) {
    const int64_t t = base + lane;
    const bool active = t < total;
    const int chunk = (int)(t % TPR);
    const int64_t row = active ? t / TPR : 0;
    float gv[8];
    if (active) {
      const float4 a = reinterpret_cast<const float4*>(g + row * kD + chunk * 8)[0];
      const float4 b2 = reinterpret_cast<const float4*>(g + row * kD + chunk * 8)[1];
      gv[0] = a.x; gv[1] = a.y; gv[2] = a.z; gv[3] = a.w;
      gv[4] = b2.x; gv[5] = b2.y; gv[6] = b2.z; gv[7] = b2.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) gv[j] = 0.f;
    }
    if (xpos && active) {
      const int n = (int)((row / H) % N);
      const float rel = (float)(n - center) * (1.f / 512.f);
      const double two_pi = 6.283185307179586476925286766559;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int i = chunk * 4 + j;
        double a = (double)n * tab.theta[i];
        a -= two_pi * rint(a * (1.0 / two_pi));
        float sn, cs;
        sincosf((float)a, &sn, &cs);
        const float e = tab.log2zeta[i] * rel;
        const float sc = exp2f(is_k ? -e : e);
        const float g0 = gv[2 * j], g1 = gv[2 * j + 1];
        gv[2 * j] = (g0 * cs + g1 * sn) * sc;
        gv[2 * j + 1] = (g1 * cs - g0 * sn) * sc;
      }
    }
    if (qk_norm) {
      float xv[8];
      if (active) {
        load8(x + row * kD + chunk * 8, xv);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) xv[j] = 0.f;
      }
      float ss = 0.f, dot = 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        ss = fmaf(xv[j], xv[j], ss);
        dot = fmaf(xv[j], gv[j], dot);
      }
#pragma unroll
      for (int m = 1; m < TPR; m <<= 1) {
        ss += __shfl_xor_sync(0xffffffffu, ss, m);
        dot += __shfl_xor_sync(0xffffffffu, dot, m);
      }
      const float nrm = sqrtf(ss);
      const float a = 1.f / fmaxf(nrm, 1e-12f);
      // <xhat, g> = a <x, g>; g - xhat <xhat, g> = g - x a^2 <x, g>
      const float c = nrm > 1e-12f ? a * a * dot : 0.f;
#pragma unroll
      for (int j = 0; j < 8; ++j) gv[j] = a * (gv[j] - xv[j] * c);
    }
    if (active) {
      reinterpret_cast<float4*>(g + row * kD + chunk * 8)[0] = make_float4(gv[0], gv[1], gv[2], gv[3]);
      reinterpret_cast<float4*>(g + row * kD + chunk * 8)[1] = make_float4(gv[4], gv[5], gv[6], gv[7]);
    }
  }
}

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

int64_t elem_bytes(int dtype) { return dtype == LONGNET_DTYPE_F32 ? 4 : 2; }

template <typename T>
int launch_typed(const Problem& p, void* qo, void* ko, const XposTable& tab, int xpos, cudaStream_t s) {
  const int64_t positions = p.B * p.N;
  const int tpr = (int)(p.D / 8);
  const int64_t threads = positions * ((p.H + kHG - 1) / kHG) * tpr;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  // at most 8 CTAs of 256 threads per SM, whole waves
  int64_t blocks = (threads + kThreads - 1) / kThreads;
  const int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  const int center = (int)(p.N / 2);
  const T* q = static_cast<const T*>(p.q);
  const T* k = static_cast<const T*>(p.k);
#define LN_PROLOGUE(TPRV)                                                                            \
  prologue_kernel<T, TPRV><<<(unsigned)blocks, kThreads, 0, s>>>(q, k, static_cast<T*>(qo),        \
                                                                 static_cast<T*>(ko), positions, (int)p.N, \
                                                                 (int)p.H, center, p.qk_norm, xpos, tab)
  switch (tpr) {
    case 2: LN_PROLOGUE(2); break;
    case 4: LN_PROLOGUE(4); break;
    case 8: LN_PROLOGUE(8); break;
    case 16: LN_PROLOGUE(16); break;
    default: return LONGNET_ERR_UNSUPPORTED;
  }
#undef LN_PROLOGUE
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

template <typename T>
int launch_bwd_typed(const Problem& p, int xpos, float* dq, float* dk, const XposTable& tab, cudaStream_t s) {
  const int64_t rows = p.B * p.N * p.H;
  const int tpr = (int)(p.D / 8);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaGetLastError();
  int64_t blocks = (rows * tpr + kThreads - 1) / kThreads;
  if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
  const int center = (int)(p.N / 2);
  for (int which = 0; which < 2; ++which) {
    const T* x = static_cast<const T*>(which ? p.k : p.q);
    float* g = which ? dk : dq;
#define LN_PROLOGUE_BWD(TPRV)                                                                               \
  prologue_bwd_kernel<T, TPRV><<<(unsigned)blocks, kThreads, 0, s>>>(x, g, rows, (int)p.N, (int)p.H, center, \
                                                                   p.qk_norm, xpos, which, tab)
    switch (tpr) {
      case 2: LN_PROLOGUE_BWD(2); break;
      case 4: LN_PROLOGUE_BWD(4); break;
      case 8: LN_PROLOGUE_BWD(8); break;
      case 16: LN_PROLOGUE_BWD(16); break;
      default: return LONGNET_ERR_UNSUPPORTED;
    }
#undef LN_PROLOGUE_BWD
    if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  }
  return LONGNET_OK;
}

XposTable make_table(int64_t D) {
  XposTable tab;
  const int n_pairs = (int)(D / 2);
  for (int i = 0; i < kMaxPairs; ++i) {
    if (i < n_pairs) {
      tab.theta[i] = pow(10000.0, -2.0 * i / (double)D);
      tab.log2zeta[i] = (float)log2((2.0 * i + 0.4 * (double)D) / (1.4 * (double)D));
    } else {
      tab.theta[i] = 0.0;
      tab.log2zeta[i] = 0.f;
    }
  }
  return tab;
}

}  // namespace

int launch_prologue_bwd(const Problem& p, int xpos, float* dq, float* dk, cudaStream_t s) {
  const XposTable tab = make_table(p.D);
  switch (p.dtype) {
    case LONGNET_DTYPE_F32: return launch_bwd_typed<float>(p, xpos, dq, dk, tab, s);
    case LONGNET_DTYPE_BF16: return launch_bwd_typed<__nv_bfloat16>(p, xpos, dq, dk, tab, s);
    case LONGNET_DTYPE_F16: return launch_bwd_typed<__half>(p, xpos, dq, dk, tab, s);
    default: return LONGNET_ERR_INVALID_ARG;
  }
}

int64_t prologue_workspace_bytes(int64_t B, int64_t N, int64_t H, int64_t D, int dtype) {
  return 2 * round_up(B * N * H * D * elem_bytes(dtype), 256);
}

// Largest |log2| of an XPOS scale over the sequence: |log2 zeta_0| times the
// farthest position from the centre, / 512 (zeta_0 = 0.4 / 1.4 is the smallest).
double xpos_max_log2_scale(int64_t N) {
  const double c = (double)(N / 2);
  const double far = c > (double)(N - 1) - c ? c : (double)(N - 1) - c;
  return -log2(0.4 / 1.4) * far / 512.0;
}

bool prologue_supports(const Problem& p, int xpos) {
  if (p.D % 16 != 0 || p.D > 128) return false;
  if (p.N > ((int64_t)1 << 30)) return false;
  if (xpos) {
    // the scaled rows must stay in the input format's normal range
    const double lim = p.dtype == LONGNET_DTYPE_F16 ? 8.0 : 100.0;
    if (xpos_max_log2_scale(p.N) > lim) return false;
  }
  return true;
}

int launch_prologue(const Problem& p, int xpos, void* qo, void* ko, cudaStream_t s) {
  const XposTable tab = make_table(p.D);
  switch (p.dtype) {
    case LONGNET_DTYPE_F32: return launch_typed<float>(p, qo, ko, tab, xpos, s);
    case LONGNET_DTYPE_BF16: return launch_typed<__nv_bfloat16>(p, qo, ko, tab, xpos, s);
    case LONGNET_DTYPE_F16: return launch_typed<__half>(p, qo, ko, tab, xpos, s);
    default: return LONGNET_ERR_INVALID_ARG;
  }
}

}  // namespace longnet
