// Kernel family SMALLSEG: the multi-pattern dilated-attention forward when
// every pattern's segments are short (all patterns share one segment length
// W <= 64, bf16, D = 64).  Such shapes move far more bytes than they compute
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
//     mma.sync m16n8k16 (bf16 in, fp32 accumulate) and an fp32 softmax;
//   * patterns other than the r = 1 one park their normalised rows (16-byte
//     chunks rotated by row, like the TMA swizzle, so a fragment's 8 rows hit
//     distinct banks) and lse in the pair's shared memory; the r = 1 pattern, processed last, merges
//     them row by row with weights e^{lse_p} ("LONGNET: Scaling Transformer
//     to 1 billion tokens", section "Token expansion reaches 1 billion+",
//     read as the softmax-denominator-weighted combination) and the rows go
//     out as coalesced 128-byte stores.
// Warps of an SM sit at different points of their load/compute/store cycle,
// which keeps bytes in flight while others compute.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "device_util.cuh"
#include "params.h"

namespace longnet {
namespace ss {

constexpr int kD = 64;
constexpr int kMaxW = 64;
constexpr int kMaxPat = 4;
constexpr int kTile = kMaxW * kD * 2;  // 8 KB
constexpr int kSmemLimit = 232448;

struct Params {
  Problem pb;
  int W;                    // common segment length
  int order[kMaxPat];       // patterns in processing order (the r = 1 one last)
  int park_off[kMaxPat];    // byte offset of each parked pattern's rows in a pair's region
  int park_rows[kMaxPat];   // rows reserved for it (ceil(W / r))
  int pair_bytes;           // shared memory per warp pair (1024-aligned)
  int n_pairs;
  int64_t n_items;          // B * (N / W) * H
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
// D += A * B, m16n8k16, bf16 inputs, fp32 accumulators
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Byte address of the 16-byte chunk `ch` of row `row` in a 128-byte-swizzled
// tile of 128-byte rows (the layout the TMA writes).
__device__ __forceinline__ uint32_t sw_addr(uint32_t base, int row, int ch) {
  return base + (uint32_t)row * 128u + ((uint32_t)(ch ^ (row & 7)) << 4);
}

// ------------------------------------------------------------ kernel

__global__ void __launch_bounds__(512, 1)
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

  const int W = P.W;
  const int64_t H = P.pb.H, N = P.pb.N;
  const int n_seg = (int)(N / W);
  const int g = lane >> 2, t4 = lane & 3;  // mma fragment coordinates
  const float scale_log2 = 1.4426950408889634f * rsqrtf((float)kD);
  const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
  __nv_bfloat16* outp = static_cast<__nv_bfloat16*>(P.pb.out);
  uint32_t phase = 0;

  for (int64_t item = (int64_t)blockIdx.x * P.n_pairs + pair; item < P.n_items;
       item += (int64_t)gridDim.x * P.n_pairs, phase ^= 1) {
    const int h = (int)(item % H);
    const int64_t bs = item / H;
    const int seg = (int)(bs % n_seg);
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
    if (!mbar_wait(bar, phase, P.wait_limit_ns)) {
      record_status(P.pb.status, kStatusTimeout);
      return;
    }

    bool ok = true;
    for (int pi = 0; pi < P.pb.n_pat; ++pi) {
      const int p = P.order[pi];
      const bool last = pi == P.pb.n_pat - 1;
      // the other warp's parked rows are complete before the merging pattern
      if (last && pi > 0 && !(ok = pair_sync())) break;
      const int r = (int)P.pb.r[p];
      const int o = h % r;
      const int m = o >= W ? 0 : (W - o + r - 1) / r;  // kept rows of this head
      if (m == 0) continue;
      const int n_kt = (m + 15) >> 4;  // 16-key steps
      uint8_t* park = region + P.park_off[p];
      float* park_l = reinterpret_cast<float*>(park + P.park_rows[p] * 128);
      for (int rc = wsub; rc < ((m + 15) >> 4); rc += 2) {
        // ---- S = Q K^T for rows [16 rc, 16 rc + 16) of the sparsified segment
        float acc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        {
          // row (sparse index) this lane addresses for the A fragments
          int qi = rc * 16 + (lane & 15);
          if (qi >= m) qi = m - 1;
          const int qrow = o + r * qi;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            uint32_t a[4];
            ldsm_x4(sw_addr(q_base, qrow, 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
            for (int np = 0; np < 4; ++np) {  // pairs of 8-key tiles
              if (np * 16 >= ((m + 15) & ~15)) break;
              // matrices: keys [16np, 16np+8) d-chunk 2kk, same keys d-chunk 2kk+1,
              // keys [16np+8, 16np+16) d-chunks 2kk, 2kk+1
              int kj = np * 16 + (lane & 7) + ((lane >> 4) << 3);
              if (kj >= m) kj = m - 1;
              const int krow = o + r * kj;
              uint32_t b0, b1, b2, b3;
              ldsm_x4(sw_addr(k_base, krow, 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
              mma16816(acc[2 * np], a, b0, b1);
              mma16816(acc[2 * np + 1], a, b2, b3);
            }
          }
        }
        // ---- softmax over the m keys (rows g and g + 8 of this chunk)
        const int row0 = rc * 16 + g, row1 = row0 + 8;
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const int c0 = nt * 8 + 2 * t4;
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int c = c0 + e;
            const bool k_ok = c < m;
            const bool ok0 = k_ok && (!P.pb.causal || c <= row0);
            const bool ok1 = k_ok && (!P.pb.causal || c <= row1);
            acc[nt][e] = ok0 ? acc[nt][e] * scale_log2 : -INFINITY;
            acc[nt][2 + e] = ok1 ? acc[nt][2 + e] * scale_log2 : -INFINITY;
            mx0 = fmaxf(mx0, acc[nt][e]);
            mx1 = fmaxf(mx1, acc[nt][2 + e]);
          }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        if (mx0 == -INFINITY) mx0 = 0.f;  // padding rows past m
        if (mx1 == -INFINITY) mx1 = 0.f;
        float l0 = 0.f, l1 = 0.f;
        uint32_t pa[4][4];  // P as A fragments, one per 16-key step
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const float p0 = ex2(acc[nt][0] - mx0), p1 = ex2(acc[nt][1] - mx0);
          const float p2 = ex2(acc[nt][2] - mx1), p3 = ex2(acc[nt][3] - mx1);
          l0 += p0 + p1;
          l1 += p2 + p3;
          const int kk = nt >> 1, hi = nt & 1;
          pa[kk][hi * 2 + 0] = pack2(p0, p1);
          pa[kk][hi * 2 + 1] = pack2(p2, p3);
        }
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
        // ---- O = P V (16 rows x 64 dims)
        float ov[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) ov[nt][e] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          if (kk >= n_kt) break;
          // the A fragment of step kk: (row g, keys 16kk+2t4..), (row g+8, ..),
          // (row g, keys 16kk+8+2t4..), (row g+8, ..)
          const uint32_t a[4] = {pa[kk][0], pa[kk][1], pa[kk][2], pa[kk][3]};
          int vj = kk * 16 + (lane & 15);
          if (vj >= m) vj = m - 1;  // masked keys have P = 0
          const int vrow = o + r * vj;
#pragma unroll
          for (int dp = 0; dp < 4; ++dp) {  // pairs of 8-dim tiles
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(sw_addr(v_base, vrow, 2 * dp + (lane >> 4)), b0, b1, b2, b3);
            mma16816(ov[2 * dp], a, b0, b1);
            mma16816(ov[2 * dp + 1], a, b2, b3);
          }
        }
        // ---- normalise; park, or merge with the parked patterns and stage out
        const float inv0 = 1.f / l0, inv1 = 1.f / l1;
        float lse0 = mx0 + __log2f(l0), lse1 = mx1 + __log2f(l1);  // log2 domain
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          ov[nt][0] *= inv0;
          ov[nt][1] *= inv0;
          ov[nt][2] *= inv1;
          ov[nt][3] *= inv1;
        }
        if (!last) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int row = half ? row1 : row0;
            if (row < m) {
#pragma unroll
              for (int nt = 0; nt < 8; ++nt)
                *reinterpret_cast<uint32_t*>(park + row * 128 + ((nt ^ (row & 7)) << 4) + 4 * t4) =
                    pack2(ov[nt][2 * half], ov[nt][2 * half + 1]);
              if (t4 == 0) park_l[row] = half ? lse1 : lse0;
            }
          }
        } else {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int row = half ? row1 : row0;  // sparse index = position in segment (r = 1)
            float lse = half ? lse1 : lse0;
            if (row < m) {
              for (int qi = 0; qi < pi; ++qi) {
                const int q = P.order[qi];
                const int rq = (int)P.pb.r[q], oq = h % rq;
                const int rel = row - oq;
                if (rel < 0 || rel % rq) continue;
                const int kq = rel / rq;
                const uint8_t* pk = region + P.park_off[q];
                const float lq = reinterpret_cast<const float*>(pk + P.park_rows[q] * 128)[kq];
                const float mxl = fmaxf(lse, lq);
                const float wa = ex2(lse - mxl), wb = ex2(lq - mxl);
                const float iw = 1.f / (wa + wb);
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) {
                  const __nv_bfloat162 pv =
                      *reinterpret_cast<const __nv_bfloat162*>(pk + kq * 128 + ((nt ^ (kq & 7)) << 4) + 4 * t4);
                  ov[nt][2 * half] = (wa * ov[nt][2 * half] + wb * __bfloat162float(pv.x)) * iw;
                  ov[nt][2 * half + 1] = (wa * ov[nt][2 * half + 1] + wb * __bfloat162float(pv.y)) * iw;
                }
                lse = mxl + __log2f(wa + wb);
              }
              // stage the row over its own Q row (no longer read: later chunks
              // read other rows) in the same swizzled layout
#pragma unroll
              for (int nt = 0; nt < 8; ++nt)
                *reinterpret_cast<uint32_t*>(sQ + sw_addr(0, row, nt) + 4 * t4) =
                    pack2(ov[nt][2 * half], ov[nt][2 * half + 1]);
              if (t4 == 0 && P.pb.lse)
                P.pb.lse[((int64_t)b * H + h) * N + (int64_t)seg * W + row] = lse * 0.69314718055994531f;
            }
          }
        }
        __syncwarp();
      }
    }
    if (!ok) return;
    // ---- coalesced store of the rows this warp staged (its 16-row chunks):
    // 16-byte chunks, 8 per row
    __syncwarp();
    for (int rc = wsub; rc * 16 < W; rc += 2) {
      for (int idx = lane; idx < 16 * 8; idx += 32) {
        const int row = rc * 16 + (idx >> 3), ch = idx & 7;
        if (row >= W) break;
        const uint4 u = *reinterpret_cast<const uint4*>(sQ + sw_addr(0, row, ch));
        *reinterpret_cast<uint4*>(outp + (((int64_t)b * N + (int64_t)seg * W + row) * H + h) * kD + ch * 8) = u;
      }
    }
    if (!pair_sync()) return;
  }
}

// ------------------------------------------------------------ host side

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
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    cudaGetLastError();
  });
  return fn;
}

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
  if (p.dtype != LONGNET_DTYPE_BF16 || p.D != kD) return false;
  if (p.n_pat < 1 || p.n_pat > kMaxPat) return false;
  const int64_t W = p.w[0];
  if (W < 1 || W > kMaxW || W % 8 != 0) return false;
  for (int i = 0; i < p.n_pat; ++i)
    if (p.w[i] != W) return false;
  if (p.H > 65535 || p.B > 65535 || p.N > (int64_t)INT32_MAX) return false;
  int off[kMaxPat], rows[kMaxPat], order[kMaxPat];
  const int pb = pair_bytes(p, off, rows, order);
  return pb > 0 && pb + 1024 <= kSmemLimit;
}

int launch_smallseg(const Problem& pb, cudaStream_t stream) {
  using namespace ss;
  EncodeTiledFn enc = get_encoder();
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
  if (P.pair_bytes <= 0) return LONGNET_ERR_UNSUPPORTED;
  P.n_pairs = (kSmemLimit - 1024) / P.pair_bytes;
  if (P.n_pairs > 8) P.n_pairs = 8;
  if (P.n_pairs < 1) return LONGNET_ERR_UNSUPPORTED;
  P.n_items = pb.B * (pb.N / P.W) * pb.H;
  const void* bases[3] = {pb.q, pb.k, pb.v};
  for (int t = 0; t < 3; ++t) {
    cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)pb.H, (cuuint64_t)pb.N, (cuuint64_t)pb.B};
    cuuint64_t strides[3] = {(cuuint64_t)(kD * 2), (cuuint64_t)(pb.H * kD * 2),
                             (cuuint64_t)(pb.N * pb.H * kD * 2)};
    cuuint32_t box[4] = {(cuuint32_t)kD, 1, (cuuint32_t)P.W, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(&maps.m[t], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(bases[t]), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return LONGNET_ERR_CUDA;
  }
  int dev = 0, n_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return LONGNET_ERR_CUDA;
  static int attr_set[64] = {0};
  if (dev < 0 || dev >= 64) return LONGNET_ERR_CUDA;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(smallseg_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit) !=
        cudaSuccess)
      return LONGNET_ERR_CUDA;
    attr_set[dev] = 1;
  }
  const int smem = P.n_pairs * P.pair_bytes + 1024;
  int64_t grid = (P.n_items + P.n_pairs - 1) / P.n_pairs;
  if (grid > n_sm) grid = n_sm;
  smallseg_kernel<<<(unsigned)grid, P.n_pairs * 64, smem, stream>>>(P, maps);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

}  // namespace longnet
