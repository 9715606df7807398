// Row gather and scatter for the sequence-parallel forward.
//
// When the sequence is split over devices ("LONGNET: Scaling Transformer to
// 1 billion tokens", section "Token expansion reaches 1 billion+"; the
// two-device split of "1000000000！微软改进Transformer一次能记住这么多token了",
// section "如何做到？"), a segment longer than one device's shard spans
// several devices, and each device needs the keys and values of that
// segment's kept rows held by the others.  These two kernels move those rows
// between a tensor [B, N, H, D] (seen as rows of D elements) and a packed
// buffer that the collective exchanges: one warp per row, 16-byte accesses.
// Every index is checked against the row count it addresses; an index out of
// range records LONGNET_ERR_DEVICE_BOUNDS in the status word and its row is
// skipped.
#include <cuda_runtime.h>
#include <stdint.h>

#include "device_util.cuh"
#include "params.h"

namespace longnet {
namespace {

constexpr int kWarpsPerBlock = 8;

// dst[dst_idx(i)] = src[src_idx(i)] for i < n, rows of row16 16-byte words;
// an index array that is null means the identity.
__global__ void __launch_bounds__(kWarpsPerBlock * 32)
    move_rows_kernel(const uint4* __restrict__ src, const int64_t* __restrict__ src_idx, int64_t src_rows,
                     uint4* __restrict__ dst, const int64_t* __restrict__ dst_idx, int64_t dst_rows,
                     int64_t n, int row16, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * kWarpsPerBlock + (threadIdx.x >> 5);
  if (i >= n) return;
  const int64_t s = src_idx ? src_idx[i] : i;
  const int64_t d = dst_idx ? dst_idx[i] : i;
  if (s < 0 || s >= src_rows || d < 0 || d >= dst_rows) {
    if (lane == 0) record_status(status, kStatusBounds);
    return;
  }
  const uint4* srow = src + s * row16;
  uint4* drow = dst + d * row16;
  for (int c = lane; c < row16; c += 32) drow[c] = srow[c];
}

}  // namespace

int launch_move_rows(const void* src, const int64_t* src_idx, int64_t src_rows, void* dst,
                     const int64_t* dst_idx, int64_t dst_rows, int64_t n, int64_t row_bytes, int* status,
                     cudaStream_t stream) {
  if (n == 0) return LONGNET_OK;
  const int64_t blocks = (n + kWarpsPerBlock - 1) / kWarpsPerBlock;
  if (blocks > 0x7fffffffLL) return LONGNET_ERR_UNSUPPORTED;
  move_rows_kernel<<<(unsigned)blocks, kWarpsPerBlock * 32, 0, stream>>>(
      static_cast<const uint4*>(src), src_idx, src_rows, static_cast<uint4*>(dst), dst_idx, dst_rows, n,
      (int)(row_bytes / 16), status);
  return cudaGetLastError() == cudaSuccess ? LONGNET_OK : LONGNET_ERR_CUDA;
}

}  // namespace longnet
