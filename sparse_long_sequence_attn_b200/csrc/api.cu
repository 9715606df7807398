// C ABI of liblongnet: argument checks, kernel-family choice, status word.
//
// Everything the caller passes is checked on the host before anything is
// enqueued; the device work itself lives in the family files (simt.cu,
// tcgen05.cu, smallseg.cu).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "device_util.cuh"
#include "longnet.h"
#include "params.h"

namespace longnet {

// One status word per device: the first error a kernel of this library
// records (wait timeout, failed index check).  Cleared by
// longnet_last_device_status.
__device__ int g_status_word;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_dev_mutex;
int* g_status_addr[kMaxDevices] = {nullptr};
int g_dev_checked[kMaxDevices] = {0};  // 0 unknown, 1 ok, -1 not sm_100

// Device checks and the status word's device address, once per device.
int current_device_state(int* dev_out, int** status_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return LONGNET_ERR_NO_DEVICE;
  }
  if (dev < 0 || dev >= kMaxDevices) return LONGNET_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (g_dev_checked[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
      cudaGetLastError();
      return LONGNET_ERR_NO_DEVICE;
    }
    if (major != 10 || minor != 0) {
      g_dev_checked[dev] = -1;
    } else {
      void* addr = nullptr;
      if (cudaGetSymbolAddress(&addr, g_status_word) != cudaSuccess || addr == nullptr) {
        cudaGetLastError();
        return LONGNET_ERR_CUDA;
      }
      g_status_addr[dev] = static_cast<int*>(addr);
      g_dev_checked[dev] = 1;
    }
  }
  if (g_dev_checked[dev] != 1) return LONGNET_ERR_NO_DEVICE;
  *dev_out = dev;
  *status_out = g_status_addr[dev];
  return LONGNET_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Argument checks common to every family; fills the problem block.
int check_args(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B,
               int64_t N, int64_t H, int64_t D, int n_pat, const int64_t* w, const int64_t* r,
               int causal, int dtype, Problem* pb) {
  if (!q || !k || !v || !out) return LONGNET_ERR_INVALID_ARG;
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0) return LONGNET_ERR_INVALID_ARG;
  if (N > (int64_t)INT32_MAX || H > 65535 || D > 65535) return LONGNET_ERR_INVALID_ARG;
  if (B > (int64_t)1 << 40 || B * N > ((int64_t)1 << 40) || B * N * H * D > ((int64_t)1 << 50))
    return LONGNET_ERR_INVALID_ARG;
  if (n_pat < 1 || n_pat > LONGNET_MAX_PATTERNS || !w || !r) return LONGNET_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return LONGNET_ERR_INVALID_ARG;
  if (dtype != LONGNET_DTYPE_F32 && dtype != LONGNET_DTYPE_BF16 && dtype != LONGNET_DTYPE_F16)
    return LONGNET_ERR_INVALID_ARG;
  for (int i = 0; i < n_pat; ++i) {
    if (r[i] < 1 || w[i] < 1) return LONGNET_ERR_INVALID_ARG;
  }
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return LONGNET_ERR_MISALIGNED;
  if (lse && !aligned(lse, 4)) return LONGNET_ERR_MISALIGNED;
  memset(pb, 0, sizeof(*pb));
  pb->q = q;
  pb->k = k;
  pb->v = v;
  pb->out = out;
  pb->lse = lse;
  pb->B = B;
  pb->N = N;
  pb->H = H;
  pb->D = D;
  pb->n_pat = n_pat;
  pb->causal = causal;
  pb->dtype = dtype;
  for (int i = 0; i < n_pat; ++i) {
    pb->w[i] = w[i];
    pb->r[i] = r[i];
  }
  pb->q0 = 0;
  pb->q1 = N;
  pb->h0 = 0;
  pb->h1 = H;
  return LONGNET_OK;
}

bool simt_supports(const Problem& p) { return p.D == 16 || p.D == 32 || p.D == 64 || p.D == 128; }

int choose_impl(const Problem& p) {
  if (smallseg_supports(p)) return LONGNET_IMPL_SMALLSEG;
  // The fused family first: the per-pattern one is as fast at 32K and faster
  // on longer sequences, but rounds out to the input format after every
  // pattern's merge, which on six patterns exceeds the bf16 error bound.
  if (tcgen05_supports(p)) return LONGNET_IMPL_TCGEN05;
  if (perpattern_supports(p)) return LONGNET_IMPL_PATTERNS;
  if (simt_supports(p)) return LONGNET_IMPL_SIMT;
  return LONGNET_ERR_UNSUPPORTED;
}

// The watchdog self-test: a barrier that expects one arrival which never
// comes.  The bounded wait gives up after limit_ns and records a timeout.
__global__ void watchdog_selftest_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(&bar, 0, limit_ns)) record_status(status, kStatusTimeout);
  }
  __syncthreads();
}

}  // namespace
}  // namespace longnet

using namespace longnet;

namespace longnet {
namespace {
// Launch the attention of a checked problem with the family impl (AUTO picks).
int run(Problem& pb, int impl, longnet_stream_t stream) {
  int dev = 0;
  int rc = current_device_state(&dev, &pb.status);
  if (rc) return rc;
  if (impl == LONGNET_IMPL_AUTO) {
    impl = choose_impl(pb);
    if (impl < 0) return impl;
  }
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  switch (impl) {
    case LONGNET_IMPL_SIMT:
      if (!simt_supports(pb)) return LONGNET_ERR_UNSUPPORTED;
      return launch_simt(pb, s);
    case LONGNET_IMPL_TCGEN05:
      if (!tcgen05_supports(pb)) return LONGNET_ERR_UNSUPPORTED;
      return launch_tcgen05(pb, s);
    case LONGNET_IMPL_SMALLSEG:
      if (!smallseg_supports(pb)) return LONGNET_ERR_UNSUPPORTED;
      return launch_smallseg(pb, s);
    case LONGNET_IMPL_PATTERNS:
      if (!perpattern_supports(pb)) return LONGNET_ERR_UNSUPPORTED;
      return launch_perpattern(pb, s);
    default:
      return LONGNET_ERR_INVALID_ARG;
  }
}

int check_part(Problem& pb, int64_t q0, int64_t q1, int64_t h0, int64_t h1) {
  if (q0 < 0 || q1 > pb.N || q0 >= q1 || h0 < 0 || h1 > pb.H || h0 >= h1) return LONGNET_ERR_INVALID_ARG;
  pb.q0 = q0;
  pb.q1 = q1;
  pb.h0 = h0;
  pb.h1 = h1;
  return LONGNET_OK;
}

int forward(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t N,
            int64_t H, int64_t D, int n_pat, const int64_t* w, const int64_t* r, int causal, int dtype,
            int flags, int impl, int64_t q0, int64_t q1, int64_t h0, int64_t h1, longnet_stream_t stream) {
  if (impl < LONGNET_IMPL_AUTO || impl > LONGNET_IMPL_PATTERNS || impl == LONGNET_IMPL_TILES)
    return LONGNET_ERR_INVALID_ARG;
  if (flags & ~LONGNET_FLAG_QK_NORM) return LONGNET_ERR_INVALID_ARG;
  Problem pb;
  int rc = check_args(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype, &pb);
  if (rc) return rc;
  rc = check_part(pb, q0, q1, h0, h1);
  if (rc) return rc;
  pb.qk_norm = (flags & LONGNET_FLAG_QK_NORM) ? 1 : 0;
  return run(pb, impl, stream);
}

// The forward with the q/k prologue into a caller-provided workspace.
int forward_ws(const void* q, const void* k, const void* v, void* out, float* lse, int64_t B, int64_t N,
               int64_t H, int64_t D, int n_pat, const int64_t* w, const int64_t* r, int causal, int dtype,
               int flags, int impl, void* workspace, int64_t workspace_bytes, longnet_stream_t stream) {
  if (impl < LONGNET_IMPL_AUTO || impl > LONGNET_IMPL_PATTERNS || impl == LONGNET_IMPL_TILES)
    return LONGNET_ERR_INVALID_ARG;
  if (flags & ~(LONGNET_FLAG_QK_NORM | LONGNET_FLAG_XPOS)) return LONGNET_ERR_INVALID_ARG;
  Problem pb;
  int rc = check_args(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype, &pb);
  if (rc) return rc;
  if (flags == 0) return run(pb, impl, stream);
  if (!workspace || workspace_bytes < prologue_workspace_bytes(B, N, H, D, dtype))
    return LONGNET_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return LONGNET_ERR_MISALIGNED;
  pb.qk_norm = (flags & LONGNET_FLAG_QK_NORM) ? 1 : 0;
  const int xpos = (flags & LONGNET_FLAG_XPOS) ? 1 : 0;
  if (!prologue_supports(pb, xpos)) return LONGNET_ERR_UNSUPPORTED;
  int dev = 0;
  rc = current_device_state(&dev, &pb.status);
  if (rc) return rc;
  char* qo = static_cast<char*>(workspace);
  char* ko = qo + prologue_workspace_bytes(B, N, H, D, dtype) / 2;
  rc = launch_prologue(pb, xpos, qo, ko, reinterpret_cast<cudaStream_t>(stream));
  if (rc) return rc;
  pb.q = qo;
  pb.k = ko;
  pb.qk_norm = 0;
  return run(pb, impl, stream);
}
}  // namespace
}  // namespace longnet

extern "C" int longnet_dilated_attn_fwd_ex(const void* q, const void* k, const void* v,
                                           void* out, float* lse, int64_t B, int64_t N, int64_t H,
                                           int64_t D, int n_pat, const int64_t* w, const int64_t* r,
                                           int causal, int dtype, int flags, int impl,
                                           longnet_stream_t stream) {
  return forward(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype, flags, impl, 0, N, 0, H,
                 stream);
}

extern "C" int64_t longnet_fwd_workspace_bytes(int64_t B, int64_t N, int64_t H, int64_t D, int dtype,
                                               int flags) {
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0 || B * N > ((int64_t)1 << 40) || H > 65535 || D > 65535 ||
      B * N * H * D > ((int64_t)1 << 50))
    return LONGNET_ERR_INVALID_ARG;
  if (dtype != LONGNET_DTYPE_F32 && dtype != LONGNET_DTYPE_BF16 && dtype != LONGNET_DTYPE_F16)
    return LONGNET_ERR_INVALID_ARG;
  if (flags & ~(LONGNET_FLAG_QK_NORM | LONGNET_FLAG_XPOS)) return LONGNET_ERR_INVALID_ARG;
  return flags ? prologue_workspace_bytes(B, N, H, D, dtype) : 0;
}

extern "C" int longnet_dilated_attn_fwd_ws(const void* q, const void* k, const void* v, void* out,
                                           float* lse, int64_t B, int64_t N, int64_t H, int64_t D,
                                           int n_pat, const int64_t* w, const int64_t* r, int causal,
                                           int dtype, int flags, int impl, void* workspace,
                                           int64_t workspace_bytes, longnet_stream_t stream) {
  return forward_ws(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype, flags, impl, workspace,
                    workspace_bytes, stream);
}

namespace longnet {
namespace {
// The fixed workspace of longnet_dilated_attn_fwd_noalloc, for callers that
// cannot allocate device memory at the call (a C host without a device
// allocator, a process whose device memory is planned up front): part of the
// library's own device memory, so the call allocates nothing.  Its device
// address is looked up once per device, with that device current.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LONGNET_NOALLOC_SCRATCH_BYTES];
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {nullptr};

int noalloc_scratch(void** addr) {
  int dev = 0;
  int* status = nullptr;
  int rc = current_device_state(&dev, &status);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return LONGNET_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *addr = g_noalloc_addr[dev];
  return LONGNET_OK;
}
}  // namespace
}  // namespace longnet

extern "C" int longnet_dilated_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* out,
                                                float* lse, int64_t B, int64_t N, int64_t H, int64_t D,
                                                int n_pat, const int64_t* w, const int64_t* r, int causal,
                                                int dtype, int flags, int impl, longnet_stream_t stream) {
  void* scratch = nullptr;
  if (flags != 0) {
    const int64_t need = longnet_fwd_workspace_bytes(B, N, H, D, dtype, flags);
    if (need < 0) return (int)need;
    if (need > (int64_t)LONGNET_NOALLOC_SCRATCH_BYTES) return LONGNET_ERR_SCRATCH_LIMIT;
    const int rc = noalloc_scratch(&scratch);
    if (rc) return rc;
  }
  return forward_ws(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype, flags, impl, scratch,
                    LONGNET_NOALLOC_SCRATCH_BYTES, stream);
}

namespace longnet {
namespace {
// Copy streams and events of the host-buffer forward, per device, created on
// its first call on that device.  The events are reused from call to call:
// calls are enqueued one at a time (g_pipe_mutex), and a wait takes the
// state of an event's latest record at the time the wait is enqueued.
constexpr int kMaxChunks = 64;
struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, out_done = nullptr;
  cudaEvent_t in_done[kMaxChunks] = {};
  cudaEvent_t comp_done[kMaxChunks] = {};
};
std::mutex g_pipe_mutex;
HostPipe g_pipe[kMaxDevices];

int host_pipe(int dev, HostPipe** out) {
  HostPipe& hp = g_pipe[dev];
  if (!hp.ready) {
    bool ok = cudaStreamCreateWithFlags(&hp.in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&hp.out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&hp.out_done, cudaEventDisableTiming) == cudaSuccess;
    for (int c = 0; ok && c < kMaxChunks; ++c)
      ok = cudaEventCreateWithFlags(&hp.in_done[c], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&hp.comp_done[c], cudaEventDisableTiming) == cudaSuccess;
    if (!ok) {
      cudaGetLastError();
      return LONGNET_ERR_CUDA;  // what was created stays for the next attempt to replace
    }
    hp.ready = true;
  }
  *out = &hp;
  return LONGNET_OK;
}

int elem_bytes(int dtype) { return dtype == LONGNET_DTYPE_F32 ? 4 : 2; }
}  // namespace
}  // namespace longnet

extern "C" int longnet_dilated_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                                             void* out_host, float* lse_host, void* q_dev, void* k_dev,
                                             void* v_dev, void* out_dev, float* lse_dev, int64_t B,
                                             int64_t N, int64_t H, int64_t D, int n_pat, const int64_t* w,
                                             const int64_t* r, int causal, int dtype, int flags, int impl,
                                             int64_t pieces, longnet_stream_t stream) {
  using namespace longnet;
  // every argument first, on the host: nothing is enqueued for a bad call
  if (!q_host || !k_host || !v_host || !out_host || (lse_host && !lse_dev)) return LONGNET_ERR_INVALID_ARG;
  if (pieces < 0) return LONGNET_ERR_INVALID_ARG;
  if (impl < LONGNET_IMPL_AUTO || impl > LONGNET_IMPL_PATTERNS || impl == LONGNET_IMPL_TILES)
    return LONGNET_ERR_INVALID_ARG;
  if (flags & ~LONGNET_FLAG_QK_NORM) return LONGNET_ERR_INVALID_ARG;
  Problem pb;
  int rc = check_args(q_dev, k_dev, v_dev, out_dev, lse_dev, B, N, H, D, n_pat, w, r, causal, dtype, &pb);
  if (rc) return rc;
  // How the work is cut (each piece: copy in, attend, copy out):
  //  * B >= 2: ranges of batches (independent, contiguous in memory);
  //  * B = 1, H >= 4 or not causal: ranges of heads (each head attends with
  //    its own rows), copied as strided 2-D blocks; every piece has the same
  //    work, so the last one, whose attention and copy out are not hidden,
  //    is short;
  //  * B = 1, H < 4, causal: ranges of positions, in order (a row's keys are
  //    at or before it, so they arrived with its piece or an earlier one),
  //    each attended as a part of the forward.
  int mode;  // 0 batches, 1 positions, 2 heads
  int64_t per, n_pieces;
  if (B >= 2) {
    mode = 0;
    n_pieces = pieces > 0 ? pieces : 8;
    if (n_pieces > B) n_pieces = B;
    per = (B + n_pieces - 1) / n_pieces;
  } else if (H < 4 && causal) {
    mode = 1;
    n_pieces = pieces > 0 ? pieces : 8;
    per = (N + n_pieces - 1) / n_pieces;
    per = (per + 255) / 256 * 256;  // whole 256-position blocks
  } else {
    mode = 2;
    n_pieces = pieces > 0 ? pieces : 6;
    if (n_pieces > H) n_pieces = H;
    per = (H + n_pieces - 1) / n_pieces;
  }
  const int64_t extent = mode == 0 ? B : mode == 1 ? N : H;
  if (per > extent) per = extent;
  if ((extent + per - 1) / per > kMaxChunks) per = (extent + kMaxChunks - 1) / kMaxChunks;
  n_pieces = (extent + per - 1) / per;
  int dev = 0;
  int* status = nullptr;
  rc = current_device_state(&dev, &status);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(g_pipe_mutex);
  HostPipe* hp = nullptr;
  rc = host_pipe(dev, &hp);
  if (rc) return rc;
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  const size_t eb = (size_t)elem_bytes(dtype);
  const size_t row = (size_t)H * (size_t)D * eb;  // one position of all heads
  auto cu = [](cudaError_t e) { return e == cudaSuccess; };
  auto at = [](const void* base, size_t off) { return static_cast<const char*>(base) + off; };
  auto atw = [](void* base, size_t off) { return static_cast<char*>(base) + off; };
  // the copies start after the work already on the caller's stream (an
  // earlier call may still read these device buffers)
  bool ok = cu(cudaEventRecord(hp->start, cs)) && cu(cudaStreamWaitEvent(hp->in, hp->start, 0)) &&
            cu(cudaStreamWaitEvent(hp->out, hp->start, 0));
  if (ok && mode == 1 && per < N) {
    // A piece's attention may read key and value rows past its end (a tile's
    // K/V block reaches further and masks them), which later pieces bring
    // in: until then they must be finite, so they start as zeros (B = 1).
    const size_t tail = (size_t)(N - per) * row;
    ok = cu(cudaMemsetAsync(atw(k_dev, (size_t)per * row), 0, tail, hp->in)) &&
         cu(cudaMemsetAsync(atw(v_dev, (size_t)per * row), 0, tail, hp->in));
  }
  int frc = LONGNET_OK;
  const void* hin[3] = {q_host, k_host, v_host};
  void* din[3] = {q_dev, k_dev, v_dev};
  for (int64_t c = 0; ok && frc == LONGNET_OK && c < n_pieces; ++c) {
    const int64_t a0 = c * per, a1 = a0 + per < extent ? a0 + per : extent;
    // the piece as a box: batches [b0, b1), positions [n0, n1), heads [h0, h1)
    const int64_t b0 = mode == 0 ? a0 : 0, b1 = mode == 0 ? a1 : B;
    const int64_t n0 = mode == 1 ? a0 : 0, n1 = mode == 1 ? a1 : N;
    const int64_t h0 = mode == 2 ? a0 : 0, h1 = mode == 2 ? a1 : H;
    // in memory: `rows` rows of `width` bytes, `pitch` apart, from byte `off`
    const size_t off = ((size_t)b0 * (size_t)N + (size_t)n0) * row + (size_t)h0 * (size_t)D * eb;
    const size_t width = (size_t)(h1 - h0) * (size_t)D * eb;
    const size_t rows = (size_t)(b1 - b0) * (size_t)(n1 - n0);
    for (int t = 0; ok && t < 3; ++t)
      ok = mode == 2 ? cu(cudaMemcpy2DAsync(atw(din[t], off), row, at(hin[t], off), row, width, rows,
                                            cudaMemcpyHostToDevice, hp->in))
                     : cu(cudaMemcpyAsync(atw(din[t], off), at(hin[t], off), rows * row, cudaMemcpyHostToDevice,
                                          hp->in));
    ok = ok && cu(cudaEventRecord(hp->in_done[c], hp->in)) && cu(cudaStreamWaitEvent(cs, hp->in_done[c], 0));
    if (!ok) break;
    // the batches of the piece as a problem of their own (B' = b1 - b0)
    const size_t boff = (size_t)b0 * (size_t)N * row;
    frc = forward(at(q_dev, boff), at(k_dev, boff), at(v_dev, boff), atw(out_dev, boff),
                  lse_dev ? lse_dev + b0 * H * N : nullptr, b1 - b0, N, H, D, n_pat, w, r, causal, dtype, flags,
                  impl, n0, n1, h0, h1, stream);
    if (frc != LONGNET_OK) break;
    ok = cu(cudaEventRecord(hp->comp_done[c], cs)) && cu(cudaStreamWaitEvent(hp->out, hp->comp_done[c], 0));
    ok = ok && (mode == 2 ? cu(cudaMemcpy2DAsync(atw(out_host, off), row, at(out_dev, off), row, width, rows,
                                                 cudaMemcpyDeviceToHost, hp->out))
                          : cu(cudaMemcpyAsync(atw(out_host, off), at(out_dev, off), rows * row,
                                               cudaMemcpyDeviceToHost, hp->out)));
    if (ok && lse_host) {
      // lse [B, H, N]: (b1 - b0) * (h1 - h0) runs of (n1 - n0) values; one
      // 2-D copy per batch
      for (int64_t b = b0; ok && b < b1; ++b) {
        const size_t lo = ((size_t)b * (size_t)H + (size_t)h0) * (size_t)N + (size_t)n0;
        ok = cu(cudaMemcpy2DAsync(lse_host + lo, (size_t)N * 4, lse_dev + lo, (size_t)N * 4,
                                  (size_t)(n1 - n0) * 4, (size_t)(h1 - h0), cudaMemcpyDeviceToHost, hp->out));
      }
    }
  }
  // the caller's stream waits for the last copies, whatever happened above,
  // so the copy streams never run ahead of it into a later call
  const bool joined = cu(cudaEventRecord(hp->out_done, hp->out)) && cu(cudaStreamWaitEvent(cs, hp->out_done, 0)) &&
                      cu(cudaEventRecord(hp->out_done, hp->in)) && cu(cudaStreamWaitEvent(cs, hp->out_done, 0));
  if (!ok || !joined) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  return frc;
}

extern "C" int longnet_dilated_attn_fwd_part(const void* q, const void* k, const void* v,
                                             void* out, float* lse, int64_t B, int64_t N,
                                             int64_t H, int64_t D, int n_pat, const int64_t* w,
                                             const int64_t* r, int causal, int dtype, int flags,
                                             int impl, int64_t q_begin, int64_t q_end,
                                             int64_t h_begin, int64_t h_end,
                                             longnet_stream_t stream) {
  return forward(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype, flags, impl, q_begin,
                 q_end, h_begin, h_end, stream);
}

namespace longnet {
namespace {
int move_rows(const void* src, const int64_t* src_idx, int64_t src_rows, void* dst, const int64_t* dst_idx,
              int64_t dst_rows, int64_t n, int64_t row_bytes, longnet_stream_t stream) {
  if (n < 0 || src_rows < 0 || dst_rows < 0 || row_bytes <= 0 || row_bytes % 16 != 0 ||
      row_bytes > ((int64_t)1 << 20))
    return LONGNET_ERR_INVALID_ARG;
  if (n == 0) return LONGNET_OK;
  if (!src || !dst || (!src_idx && !dst_idx)) return LONGNET_ERR_INVALID_ARG;
  if (!aligned(src, 16) || !aligned(dst, 16) || (src_idx && !aligned(src_idx, 8)) ||
      (dst_idx && !aligned(dst_idx, 8)))
    return LONGNET_ERR_MISALIGNED;
  int dev = 0;
  int* status = nullptr;
  int rc = current_device_state(&dev, &status);
  if (rc) return rc;
  return launch_move_rows(src, src_idx, src_rows, dst, dst_idx, dst_rows, n, row_bytes, status,
                          reinterpret_cast<cudaStream_t>(stream));
}
}  // namespace
}  // namespace longnet

extern "C" int longnet_gather_rows(const void* src, int64_t src_rows, const int64_t* idx, int64_t n,
                                   void* dst, int64_t row_bytes, longnet_stream_t stream) {
  return move_rows(src, idx, src_rows, dst, nullptr, n, n, row_bytes, stream);
}

extern "C" int longnet_scatter_rows(const void* src, int64_t n, const int64_t* idx, void* dst,
                                    int64_t dst_rows, int64_t row_bytes, longnet_stream_t stream) {
  return move_rows(src, nullptr, n, dst, idx, dst_rows, n, row_bytes, stream);
}

extern "C" int longnet_dilated_attn_fwd_impl(const void* q, const void* k, const void* v,
                                             void* out, float* lse, int64_t B, int64_t N,
                                             int64_t H, int64_t D, int n_pat, const int64_t* w,
                                             const int64_t* r, int causal, int dtype, int impl,
                                             longnet_stream_t stream) {
  return longnet_dilated_attn_fwd_ex(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype, 0,
                                     impl, stream);
}

extern "C" int longnet_dilated_attn_fwd(const void* q, const void* k, const void* v, void* out,
                                        float* lse, int64_t B, int64_t N, int64_t H, int64_t D,
                                        int n_pat, const int64_t* w, const int64_t* r, int causal,
                                        int dtype, longnet_stream_t stream) {
  return longnet_dilated_attn_fwd_impl(q, k, v, out, lse, B, N, H, D, n_pat, w, r, causal, dtype,
                                       LONGNET_IMPL_AUTO, stream);
}

extern "C" int longnet_dilated_attn_bwd(const void* q, const void* k, const void* v,
                                        const void* out, const float* lse, const void* dout,
                                        float* dq, float* dk, float* dv, int64_t B, int64_t N,
                                        int64_t H, int64_t D, int n_pat, const int64_t* w,
                                        const int64_t* r, int causal, int dtype, int flags,
                                        int impl, longnet_stream_t stream) {
  if (flags & ~LONGNET_FLAG_QK_NORM) return LONGNET_ERR_INVALID_ARG;
  if (impl != LONGNET_IMPL_AUTO && impl != LONGNET_IMPL_SIMT && impl != LONGNET_IMPL_TILES &&
      impl != LONGNET_IMPL_TCGEN05)
    return LONGNET_ERR_INVALID_ARG;
  if (!out || !lse || !dout || !dq || !dk || !dv) return LONGNET_ERR_INVALID_ARG;
  Problem pb;
  // the forward's checks on q, k, v and the shape (dq stands in the output's
  // place, the gradients go through BwdArgs); lse is read, not written
  int rc = check_args(q, k, v, dq, const_cast<float*>(lse), B, N, H, D, n_pat, w, r, causal, dtype,
                      &pb);
  if (rc) return rc;
  if (!aligned(out, 16) || !aligned(dout, 16) || !aligned(dk, 16) || !aligned(dv, 16))
    return LONGNET_ERR_MISALIGNED;
  pb.qk_norm = (flags & LONGNET_FLAG_QK_NORM) ? 1 : 0;
  if (impl == LONGNET_IMPL_AUTO && !backward_supports(pb) && !tile_backward_supports(pb))
    return LONGNET_ERR_UNSUPPORTED;
  if (impl == LONGNET_IMPL_SIMT && !backward_supports(pb)) return LONGNET_ERR_UNSUPPORTED;
  if (impl == LONGNET_IMPL_TILES && !tile_backward_supports(pb)) return LONGNET_ERR_UNSUPPORTED;
  if (impl == LONGNET_IMPL_TCGEN05 && !tcgen05_backward_supports(pb)) return LONGNET_ERR_UNSUPPORTED;
  int dev = 0;
  rc = current_device_state(&dev, &pb.status);
  if (rc) return rc;
  BwdArgs g;
  g.out = out;
  g.dout = dout;
  g.dq = dq;
  g.dk = dk;
  g.dv = dv;
  return launch_backward(pb, g, impl, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" int longnet_dilated_attn_bwd_ws(const void* q, const void* k, const void* v, const void* out,
                                           const float* lse, const void* dout, float* dq, float* dk,
                                           float* dv, int64_t B, int64_t N, int64_t H, int64_t D, int n_pat,
                                           const int64_t* w, const int64_t* r, int causal, int dtype,
                                           int flags, int impl, void* workspace, int64_t workspace_bytes,
                                           longnet_stream_t stream) {
  if (flags & ~(LONGNET_FLAG_QK_NORM | LONGNET_FLAG_XPOS)) return LONGNET_ERR_INVALID_ARG;
  if (flags == 0)
    return longnet_dilated_attn_bwd(q, k, v, out, lse, dout, dq, dk, dv, B, N, H, D, n_pat, w, r, causal,
                                    dtype, 0, impl, stream);
  if (impl != LONGNET_IMPL_AUTO && impl != LONGNET_IMPL_SIMT && impl != LONGNET_IMPL_TILES &&
      impl != LONGNET_IMPL_TCGEN05)
    return LONGNET_ERR_INVALID_ARG;
  if (!out || !lse || !dout || !dq || !dk || !dv) return LONGNET_ERR_INVALID_ARG;
  Problem pb;
  int rc = check_args(q, k, v, dq, const_cast<float*>(lse), B, N, H, D, n_pat, w, r, causal, dtype, &pb);
  if (rc) return rc;
  if (!aligned(out, 16) || !aligned(dout, 16) || !aligned(dk, 16) || !aligned(dv, 16))
    return LONGNET_ERR_MISALIGNED;
  if (!workspace || workspace_bytes < prologue_workspace_bytes(B, N, H, D, dtype)) return LONGNET_ERR_INVALID_ARG;
  if (!aligned(workspace, 256)) return LONGNET_ERR_MISALIGNED;
  pb.qk_norm = (flags & LONGNET_FLAG_QK_NORM) ? 1 : 0;
  const int xpos = (flags & LONGNET_FLAG_XPOS) ? 1 : 0;
  if (!prologue_supports(pb, xpos)) return LONGNET_ERR_UNSUPPORTED;
  // the attention's backward runs on the encoded rows, without options
  Problem enc = pb;
  char* qo = static_cast<char*>(workspace);
  char* ko = qo + prologue_workspace_bytes(B, N, H, D, dtype) / 2;
  enc.q = qo;
  enc.k = ko;
  enc.qk_norm = 0;
  if (impl == LONGNET_IMPL_AUTO && !backward_supports(enc) && !tile_backward_supports(enc))
    return LONGNET_ERR_UNSUPPORTED;
  if (impl == LONGNET_IMPL_SIMT && !backward_supports(enc)) return LONGNET_ERR_UNSUPPORTED;
  if (impl == LONGNET_IMPL_TILES && !tile_backward_supports(enc)) return LONGNET_ERR_UNSUPPORTED;
  if (impl == LONGNET_IMPL_TCGEN05 && !tcgen05_backward_supports(enc)) return LONGNET_ERR_UNSUPPORTED;
  int dev = 0;
  rc = current_device_state(&dev, &pb.status);
  if (rc) return rc;
  enc.status = pb.status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  rc = launch_prologue(pb, xpos, qo, ko, s);
  if (rc) return rc;
  BwdArgs g;
  g.out = out;
  g.dout = dout;
  g.dq = dq;
  g.dk = dk;
  g.dv = dv;
  rc = launch_backward(enc, g, impl, s);
  if (rc) return rc;
  return launch_prologue_bwd(pb, xpos, dq, dk, s);
}

extern "C" int longnet_select_impl(int64_t B, int64_t N, int64_t H, int64_t D, int n_pat,
                                   const int64_t* w, const int64_t* r, int causal, int dtype) {
  // Stand-in pointers: only their alignment (and, for lse, presence) is
  // looked at here; the call is taken as one that asks for lse.
  static __align__(16) char dummy[16];
  Problem pb;
  int rc = check_args(dummy, dummy, dummy, dummy, reinterpret_cast<float*>(dummy), B, N, H, D, n_pat, w, r,
                      causal, dtype, &pb);
  if (rc) return rc;
  return choose_impl(pb);
}

extern "C" int longnet_last_device_status(longnet_stream_t stream) {
  int dev = 0;
  int* addr = nullptr;
  int rc = current_device_state(&dev, &addr);
  if (rc) return rc;
  if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_status_word, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status_word, &zero, sizeof(int)) != cudaSuccess) {
    cudaGetLastError();
    return LONGNET_ERR_CUDA;
  }
  return word;
}

extern "C" int longnet_watchdog_selftest(int64_t limit_ns, longnet_stream_t stream) {
  int dev = 0;
  int* addr = nullptr;
  int rc = current_device_state(&dev, &addr);
  if (rc) return rc;
  if (limit_ns < 1000) limit_ns = 1000;
  if (limit_ns > 1000000000) limit_ns = 1000000000;
  watchdog_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      addr, static_cast<uint64_t>(limit_ns));
  if (cudaGetLastError() != cudaSuccess) return LONGNET_ERR_CUDA;
  return LONGNET_OK;
}

extern "C" const char* longnet_status_string(int status) {
  switch (status) {
    case LONGNET_OK: return "ok";
    case LONGNET_ERR_INVALID_ARG: return "invalid argument";
    case LONGNET_ERR_UNSUPPORTED: return "unsupported shape or dtype for this kernel family";
    case LONGNET_ERR_MISALIGNED: return "pointer misaligned";
    case LONGNET_ERR_CUDA: return "CUDA call failed";
    case LONGNET_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case LONGNET_ERR_DEVICE_BOUNDS: return "device index check failed";
    case LONGNET_ERR_NO_DEVICE: return "no usable sm_100 device";
    case LONGNET_ERR_SCRATCH_LIMIT:
      return "problem too large for the fixed scratch of longnet_dilated_attn_fwd_noalloc";
    default: return "unknown status";
  }
}

extern "C" const char* longnet_version(void) { return "longnet-b200 1.0 sm_100a"; }
