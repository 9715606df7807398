// Host/device parameter block shared by the kernels of liblongnet.
#pragma once

#include <stdint.h>

#include "longnet.h"

namespace longnet {

// One call's arguments after validation.  Pattern arrays are copied in so a
// kernel can read them from its parameter space.
struct Problem {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;  // may be null
  int64_t B, N, H, D;
  int n_pat;
  int causal;
  int dtype;
  int qk_norm;  // 1: q and k rows are scaled to unit L2 norm first (LONGNET_FLAG_QK_NORM)
  // The part of the output computed: positions [q0, q1) and heads [h0, h1)
  // (the whole output: 0, N, 0, H).  Keys and values are read wherever the
  // method needs them, inside or outside the part.
  int64_t q0, q1, h0, h1;
  int64_t w[LONGNET_MAX_PATTERNS];
  int64_t r[LONGNET_MAX_PATTERNS];
  int* status;  // device address of this device's status word
};

// The backward's extra arguments (device pointers, [B, N, H, D]): the
// forward's output and its cotangent in the problem's dtype, and the
// gradients in fp32.
struct BwdArgs {
  const void* out;
  const void* dout;
  float* dq;
  float* dk;
  float* dv;
};

// Status codes written into the device status word (first error wins).
constexpr int kStatusTimeout = LONGNET_ERR_DEVICE_TIMEOUT;
constexpr int kStatusBounds = LONGNET_ERR_DEVICE_BOUNDS;

// Wait limit of every bounded device-side wait in the library.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

// Kernel launchers (one per family).  Return a longnet_status.
int launch_simt(const Problem& p, cudaStream_t stream);
int launch_tcgen05(const Problem& p, cudaStream_t stream);
int launch_smallseg(const Problem& p, cudaStream_t stream);
int launch_backward(const Problem& p, const BwdArgs& g, int impl, cudaStream_t stream);

// The q/k prologue (qk_norm and XPOS) into a workspace of
// prologue_workspace_bytes: q rows first, k rows from half of it on.
int64_t prologue_workspace_bytes(int64_t B, int64_t N, int64_t H, int64_t D, int dtype);
bool prologue_supports(const Problem& p, int xpos);
int launch_prologue(const Problem& p, int xpos, void* qo, void* ko, cudaStream_t stream);
// Its backward: the fp32 gradients of the encoded q and k rows, in place in
// dq and dk, become those of the original rows (p.q, p.k).
int launch_prologue_bwd(const Problem& p, int xpos, float* dq, float* dk, cudaStream_t stream);

// Row moves of the sequence-parallel exchange: dst[dst_idx[i]] = src[src_idx[i]]
// for i < n (a null index array is the identity), rows of row_bytes (a
// multiple of 16) bytes; indices checked against src_rows / dst_rows.
int launch_move_rows(const void* src, const int64_t* src_idx, int64_t src_rows, void* dst,
                     const int64_t* dst_idx, int64_t dst_rows, int64_t n, int64_t row_bytes, int* status,
                     cudaStream_t stream);

// Shape checks of the specialised families (host only, no device access).
bool tcgen05_supports(const Problem& p);
bool perpattern_supports(const Problem& p);  // the per-pattern tcgen05 forward
int launch_perpattern(const Problem& p, cudaStream_t stream);
bool smallseg_supports(const Problem& p);
bool backward_supports(const Problem& p);       // the SIMT backward
bool tile_backward_supports(const Problem& p);  // the mma.sync tile backward
bool tcgen05_backward_supports(const Problem& p);  // the tcgen05 backward
int launch_tcgen05_backward(const Problem& p, const BwdArgs& g, cudaStream_t stream);

}  // namespace longnet
