/*
 * longnet.h — C ABI of the B200 (sm_100a) multi-pattern dilated-attention
 * forward of LongNet.
 *
 * The operation ("LONGNET: Scaling Transformer to 1 billion tokens", section
 * "LongNet's attention allocation principle"; "LongNet论文精读", section
 * "Dilated Attention的工作原理"):
 *   for every pattern p = (w_p, r_p):
 *     - split the sequence into segments of w_p tokens;
 *     - in each segment head h keeps the rows at offsets o + r_p*k < w_p,
 *       with o = h mod r_p (each head has its own offset);
 *     - attend with softmax(Q K^T / sqrt(D)) V over the kept rows of the
 *       segment (causal: a kept row sees kept rows at or before itself);
 *     - put the rows back at their positions;
 *   then combine the patterns row by row, each weighted by its softmax
 *   denominator:  out = sum_p e^{lse_p} O_p / sum_p e^{lse_p},
 *   lse = log sum_p e^{lse_p}, over the patterns that keep the row (the
 *   reading adopted for "combine local attention into global attention",
 *   same page, section "Token expansion reaches 1 billion+").  A row kept by
 *   no pattern gets out = 0 and lse = -inf.
 *
 * Conventions shared by every entry point
 *   - q, k, v, out: device pointers, contiguous [B, N, H, D] in the dtype
 *     given (LONGNET_DTYPE_F32, LONGNET_DTYPE_BF16 or LONGNET_DTYPE_F16); 16-byte aligned.
 *   - lse: device pointer to fp32 [B, H, N] (natural log, scale included),
 *     or NULL when not wanted.  4-byte aligned.
 *   - w, r: HOST arrays of n_pat pattern parameters, read during the call
 *     and not kept.  1 <= n_pat <= LONGNET_MAX_PATTERNS, r >= 1, w >= 1.
 *     When w does not divide N the last segment is the shorter rest of the
 *     sequence (no padding); w > N makes one segment of the whole sequence.
 *     Patterns may repeat and come in any order; a repeated pattern counts
 *     twice.
 *   - causal: 1 = causal inside each sparsified segment, 0 = full.
 *   - stream: a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; the call returns before it finishes.
 *   - Memory: every pointer is owned by the caller.  The library allocates
 *     no device or host memory in any call.  Its global state is one status
 *     word per device (see longnet_last_device_status) and, on the host,
 *     small per-device caches in static storage (the launch set-up of the
 *     last shapes and pointers, kernel attributes), guarded for concurrent
 *     callers.
 *   - Errors: every entry point returns LONGNET_OK (0) or a negative code,
 *     never aborts, traps or exits.  Arguments are checked before anything is
 *     enqueued: a rejected call enqueues nothing.
 *   - Calls may run concurrently on different streams.
 */
#ifndef LONGNET_H_
#define LONGNET_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so the header needs no CUDA. */
typedef struct CUstream_st* longnet_stream_t;

#define LONGNET_MAX_PATTERNS 16

enum longnet_status {
  LONGNET_OK = 0,
  LONGNET_ERR_INVALID_ARG = -1,   /* a size <= 0, bad pattern, NULL tensor */
  LONGNET_ERR_UNSUPPORTED = -2,   /* a valid shape the chosen kernel lacks */
  LONGNET_ERR_MISALIGNED = -3,    /* a pointer misses its alignment */
  LONGNET_ERR_CUDA = -4,          /* a CUDA call failed (launch, config) */
  LONGNET_ERR_DEVICE_TIMEOUT = -5,/* a kernel wait ran out of time (status word) */
  LONGNET_ERR_DEVICE_BOUNDS = -6, /* a kernel index check failed (status word) */
  LONGNET_ERR_NO_DEVICE = -7,     /* no usable sm_100 device */
  LONGNET_ERR_SCRATCH_LIMIT = -8  /* longnet_dilated_attn_fwd_noalloc: the problem
                                     needs more than the fixed scratch holds */
};

enum longnet_dtype { LONGNET_DTYPE_F32 = 0, LONGNET_DTYPE_BF16 = 1, LONGNET_DTYPE_F16 = 2 };

/* Kernel families.  AUTO picks per shape; the others force one (tests). */
enum longnet_impl {
  LONGNET_IMPL_AUTO = 0,
  LONGNET_IMPL_SIMT = 1,     /* fp32 FMA, any D in {16,32,64,128}, every dtype */
  LONGNET_IMPL_TCGEN05 = 2,  /* bf16 or fp16, D = 64, <= 6 patterns: TMA +
                                tcgen05/TMEM flash kernel, patterns fused in
                                shared memory */
  LONGNET_IMPL_SMALLSEG = 3, /* bf16 or fp16, D = 64, all patterns one segment
                                length w <= 64 (a multiple of 8; the last
                                segment may be shorter), up to 8
                                patterns when every r divides 8, else up to
                                4; q, k, v, out 16-byte aligned: memory-bound
                                kernel, one weighted softmax per segment */
  LONGNET_IMPL_TILES = 4,    /* backward only: bf16 or fp16, D = 64, any
                                patterns: 64-row tiles of the sparsified
                                segments on mma.sync tensor cores */
  LONGNET_IMPL_PATTERNS = 5  /* forward: bf16 or fp16, D = 16, 32, 64 or 128, any number
                                of patterns, qk_norm or not, lse required with
                                more than one:
                                one tcgen05 launch per pattern, each merging its
                                rows into out and lse (initialised to 0 and
                                -inf); out is rounded to the input format
                                between patterns */
};

/*
 * longnet_dilated_attn_fwd — the forward described at the top of this file.
 * Chooses the kernel (LONGNET_IMPL_AUTO).  Returns a longnet_status.
 */
int longnet_dilated_attn_fwd(const void* q, const void* k, const void* v,
                             void* out, float* lse,
                             int64_t B, int64_t N, int64_t H, int64_t D,
                             int n_pat, const int64_t* w, const int64_t* r,
                             int causal, int dtype, longnet_stream_t stream);

/*
 * longnet_dilated_attn_fwd_impl — same operation, with the kernel family
 * forced (enum longnet_impl).  Returns LONGNET_ERR_UNSUPPORTED when that
 * family does not cover the arguments.
 */
int longnet_dilated_attn_fwd_impl(const void* q, const void* k, const void* v,
                                  void* out, float* lse,
                                  int64_t B, int64_t N, int64_t H, int64_t D,
                                  int n_pat, const int64_t* w, const int64_t* r,
                                  int causal, int dtype, int impl,
                                  longnet_stream_t stream);

/* Options of the forward (a bit set). */
enum longnet_flags {
  /* Scale every q row and every k row (over D) to unit L2 norm before the
   * scores: x / max(|x|, 1e-12), computed in fp32.  The reading adopted for
   * the qk_norm option of the DilatedAttention module ("LongNet" docs page,
   * usage example).  Through longnet_dilated_attn_fwd_ex every forward
   * family applies it inside the attention (the small-segment kernel rounds
   * the normalised rows back to the input format, the SIMT kernel keeps them
   * in fp32, the tcgen05 and per-pattern kernels scale the scores of the rows
   * as given by both inverse norms in fp32); through
   * longnet_dilated_attn_fwd_ws a prologue pass applies it and every family
   * takes the result. */
  LONGNET_FLAG_QK_NORM = 1,
  /* XPOS on q and k, the rotary position encoding with exponential scaling
   * that the use_xpos option names ("LongNet论文精读", section "Dilated
   * Attention的核心参数解析"; the pages give no formula, the published XPOS
   * definition of Sun et al., "A Length-Extrapolatable Transformer", is
   * taken).  For the element pair (2i, 2i+1) of a row at position n:
   * theta_i = 10000^(-2i/D), zeta_i = (2i + 0.4 D) / (1.4 D),
   * s = zeta_i^((n - floor(N/2)) / 512); queries become
   * s (x0 cos(n theta_i) - x1 sin(n theta_i), x1 cos(n theta_i) + x0 sin(n theta_i))
   * and keys the same with 1/s, so a score depends on the positions' difference
   * only.  Applied after the norm when both flags are set, computed in fp32
   * and rounded to the input format.  longnet_dilated_attn_fwd_ws only.  The
   * scales must stay in the input format's range: |log2 s| <= 100 (fp32,
   * bf16: N <= 56,000 or so) or <= 8 (fp16: N <= 4,500 or so), else
   * LONGNET_ERR_UNSUPPORTED. */
  LONGNET_FLAG_XPOS = 2
};

/*
 * longnet_dilated_attn_fwd_ex — the forward with options (flags, a
 * longnet_flags bit set) and an explicit kernel family (impl, as in
 * longnet_dilated_attn_fwd_impl).  flags: LONGNET_FLAG_QK_NORM or 0; any
 * other bit (LONGNET_FLAG_XPOS included): LONGNET_ERR_INVALID_ARG.
 * The two entry points above are this call with flags = 0.
 */
int longnet_dilated_attn_fwd_ex(const void* q, const void* k, const void* v,
                                void* out, float* lse,
                                int64_t B, int64_t N, int64_t H, int64_t D,
                                int n_pat, const int64_t* w, const int64_t* r,
                                int causal, int dtype, int flags, int impl,
                                longnet_stream_t stream);

/*
 * longnet_fwd_workspace_bytes — device workspace, in bytes, that
 * longnet_dilated_attn_fwd_ws needs for these sizes, dtype and flags: 0 for
 * flags = 0, else two tensors of B*N*H*D elements of dtype (the transformed
 * q and k), each rounded up to 256 bytes.  Invalid sizes, dtype or flag
 * bits: LONGNET_ERR_INVALID_ARG (negative).
 */
int64_t longnet_fwd_workspace_bytes(int64_t B, int64_t N, int64_t H, int64_t D, int dtype, int flags);

/*
 * longnet_dilated_attn_fwd_ws — the forward with the input-side options
 * (flags: LONGNET_FLAG_QK_NORM, LONGNET_FLAG_XPOS, or both) applied by a
 * prologue pass: q and k are read once, transformed (norm first, then
 * XPOS) and written to the caller's workspace, and the attention (family
 * impl, AUTO picking as for the plain forward) runs on the workspace's q
 * and k and the caller's v, both launches on `stream` in that order.  The
 * options of the DilatedAttention module ("LongNet" docs page, usage
 * example; "LongNet论文精读", section "Dilated Attention的核心参数解析").
 *   workspace: device memory owned by the caller, 256-byte aligned
 *     (else LONGNET_ERR_MISALIGNED), at least longnet_fwd_workspace_bytes
 *     bytes (else LONGNET_ERR_INVALID_ARG), overlapping none of q, k, v, out,
 *     lse; its contents on entry do not matter and on return are the
 *     transformed q and k.  Unused when flags = 0 (the call is then
 *     longnet_dilated_attn_fwd_ex with flags 0; workspace may be null).
 *   D a multiple of 16, at most 128, for the prologue; XPOS range limits as
 *   stated at LONGNET_FLAG_XPOS (LONGNET_ERR_UNSUPPORTED).  The other
 *   arguments, results and errors are those of longnet_dilated_attn_fwd_ex.
 */
int longnet_dilated_attn_fwd_ws(const void* q, const void* k, const void* v,
                                void* out, float* lse,
                                int64_t B, int64_t N, int64_t H, int64_t D,
                                int n_pat, const int64_t* w, const int64_t* r,
                                int causal, int dtype, int flags, int impl,
                                void* workspace, int64_t workspace_bytes,
                                longnet_stream_t stream);

/* Size of the fixed device scratch of longnet_dilated_attn_fwd_noalloc, per
 * device: 32 MiB. */
#define LONGNET_NOALLOC_SCRATCH_BYTES (32 << 20)

/*
 * longnet_dilated_attn_fwd_noalloc — longnet_dilated_attn_fwd_ws with its
 * workspace taken from a fixed array of LONGNET_NOALLOC_SCRATCH_BYTES in the
 * library's own device memory (one per device) instead of from the caller.
 * The pages have no counterpart: the method says nothing about who owns
 * memory.  It is for callers that cannot allocate device memory when they
 * call: a C host with no device allocator of its own, or a serving process
 * whose device memory is planned up front (handed to its caches), where an
 * allocation at call time fails or must first free cached blocks.  The call
 * allocates nothing (no cudaMalloc or cudaFree, directly or through torch).
 *   Limit: longnet_fwd_workspace_bytes(B, N, H, D, dtype, flags) must not
 *     exceed LONGNET_NOALLOC_SCRATCH_BYTES (for bf16: B*N*H*D up to 8 Mi
 *     elements), else LONGNET_ERR_SCRATCH_LIMIT and nothing is launched.
 *     flags = 0 needs no scratch (the call is the plain forward).
 *   Contents: nothing in the scratch has to start at zero or at any value:
 *     the prologue writes every byte of it that the attention then reads.
 *   First call on a device: it looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current), which may load the
 *     library's device code; make that first call before any stream capture
 *     begins.  A failed lookup returns LONGNET_ERR_CUDA.
 *   Calls that overlap race: every call on a device uses the same array, so
 *     two calls whose work may run at the same time (different streams, or
 *     different host threads, without an ordering between them) corrupt each
 *     other's q and k.  Order them (one stream, or events).
 * The other arguments, results and errors are those of
 * longnet_dilated_attn_fwd_ws.
 */
int longnet_dilated_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                     void* out, float* lse,
                                     int64_t B, int64_t N, int64_t H, int64_t D,
                                     int n_pat, const int64_t* w, const int64_t* r,
                                     int causal, int dtype, int flags, int impl,
                                     longnet_stream_t stream);

/*
 * longnet_dilated_attn_fwd_host — the forward on inputs and outputs in HOST
 * memory, with the host<->device copies overlapped with the attention.  The
 * pages have no counterpart (they say nothing about where a model's tensors
 * live); it is the call of a host program whose q, k, v come from, and whose
 * out goes back to, host memory.  The work is cut into pieces that are
 * pipelined: the copy in of piece c + 1 runs while piece c is attended and
 * piece c - 1 is copied out.  The cut follows the method's independences:
 *   B >= 2: ranges of batches (each batch attends on its own);
 *   B = 1 and H >= 4, or not causal: ranges of heads (each head attends with
 *     its own rows), copied as strided 2-D blocks;
 *   B = 1, H < 4, causal: ranges of positions, in order (a row attends to
 *     keys at or before it, which arrived with its piece or an earlier one),
 *     each attended as a part (longnet_dilated_attn_fwd_part); the rows of
 *     k_dev and v_dev past the first piece are zeroed before any copy, since
 *     a part may read later key rows (masked) that must be finite.
 *   q_host, k_host, v_host: [B, N, H, D] inputs in host memory; out_host
 *     [B, N, H, D] and lse_host [B, H, N] (may be NULL) outputs in host
 *     memory.  Page-locked (pinned) memory lets the copies run asynchronously;
 *     pageable memory works but each copy then waits on the host.
 *   q_dev, k_dev, v_dev, out_dev: device buffers of the same shape, and
 *     lse_dev [B, H, N] (required when lse_host is given), owned by the
 *     caller and used as the copies' staging; the call allocates nothing.
 *     Their alignment rules are those of longnet_dilated_attn_fwd.
 *   pieces: how many pieces (0 = 8 ranges of batches or positions, 6 of
 *     heads); never more than the batches, positions (in blocks of 256) or
 *     heads there are, nor more than 64.
 *   flags: 0 or LONGNET_FLAG_QK_NORM (applied inside the kernels that take
 *     it, as in longnet_dilated_attn_fwd_ex); impl: as there.
 *   stream: the call enqueues on `stream` and on two copy streams of its own;
 *     the copies start after the work already on `stream`, and `stream`
 *     waits for the last copies before anything enqueued on it later, so
 *     synchronising `stream` means out_host and lse_host hold the results.
 *     The call returns once everything is enqueued.
 *   First call on a device: it creates the two copy streams and their events
 *     (kept for later calls); make that first call before any stream capture
 *     begins.  Calls are enqueued one at a time (a lock), so several host
 *     threads may call; their copies and kernels are then ordered only by
 *     their streams.
 * Returns LONGNET_ERR_INVALID_ARG for a NULL host pointer, lse_host without
 * lse_dev, pieces < 0 or any argument the plain forward rejects (checked
 * before anything is enqueued); LONGNET_ERR_CUDA when a copy cannot be
 * enqueued; otherwise the status of the first piece's forward that failed.
 */
int longnet_dilated_attn_fwd_host(const void* q_host, const void* k_host, const void* v_host,
                                  void* out_host, float* lse_host,
                                  void* q_dev, void* k_dev, void* v_dev, void* out_dev, float* lse_dev,
                                  int64_t B, int64_t N, int64_t H, int64_t D,
                                  int n_pat, const int64_t* w, const int64_t* r,
                                  int causal, int dtype, int flags, int impl,
                                  int64_t pieces, longnet_stream_t stream);

/*
 * longnet_dilated_attn_fwd_part — the forward with options and a family (as
 * longnet_dilated_attn_fwd_ex), computing only part of the output: positions
 * [q_begin, q_end) and heads [h_begin, h_end) of out and lse; every other
 * element of out and lse is left untouched.  q, k, v are full-length
 * [B, N, H, D] tensors.  The caller provides q at the part's positions and
 * heads, and k and v wherever the part's rows need keys (the kept rows of
 * the same segments, before each row when causal).  Other rows of q may hold
 * anything (rows are computed independently).  Other rows of k and v may be
 * read too, and masked: they must hold finite values, since a masked row's
 * weight, 0, multiplies its v row (zero is the natural fill).
 * This is the step a device takes when the sequence is split over devices
 * ("LONGNET: Scaling Transformer to 1 billion tokens", section "Token
 * expansion reaches 1 billion+": each device attends for its own shard,
 * the keys and values of longer segments coming from the other devices), and
 * the step of a split by heads.  0 <= q_begin < q_end <= N and
 * 0 <= h_begin < h_end <= H, else LONGNET_ERR_INVALID_ARG.  The small-segment
 * kernel takes parts made of whole segments only (the sequence's shorter last
 * one included; AUTO otherwise picks another family).  The other conventions are those of the full forward.
 */
int longnet_dilated_attn_fwd_part(const void* q, const void* k, const void* v,
                                  void* out, float* lse,
                                  int64_t B, int64_t N, int64_t H, int64_t D,
                                  int n_pat, const int64_t* w, const int64_t* r,
                                  int causal, int dtype, int flags, int impl,
                                  int64_t q_begin, int64_t q_end,
                                  int64_t h_begin, int64_t h_end,
                                  longnet_stream_t stream);

/*
 * longnet_gather_rows / longnet_scatter_rows — the data movement of the
 * sequence-parallel exchange (same pages and sections as
 * longnet_dilated_attn_fwd_part): the kept rows of one device's shard that
 * other devices need are packed into a contiguous buffer, exchanged by a
 * collective, and written back at their positions on the receiving device.
 *   gather:  dst[i] = src[idx[i]] for i < n (dst holds n rows);
 *   scatter: dst[idx[i]] = src[i] for i < n (src holds n rows).
 * A row is row_bytes bytes (a positive multiple of 16, at most 1 MiB); for a
 * [B, N, H, D] tensor the row of (b, x, h) is (b N + x) H + h and
 * row_bytes = D times the element size.  src, dst: device pointers,
 * 16-byte aligned; idx: a device array of n int64, 8-byte aligned, caller
 * owned.  src_rows / dst_rows: rows the indexed buffer holds; an index
 * outside [0, rows) is not accessed and records LONGNET_ERR_DEVICE_BOUNDS in
 * the status word (see longnet_last_device_status).  n = 0 does nothing.
 * Enqueued on stream; returns a longnet_status.
 */
int longnet_gather_rows(const void* src, int64_t src_rows, const int64_t* idx, int64_t n,
                        void* dst, int64_t row_bytes, longnet_stream_t stream);
int longnet_scatter_rows(const void* src, int64_t n, const int64_t* idx, void* dst,
                         int64_t dst_rows, int64_t row_bytes, longnet_stream_t stream);

/*
 * longnet_dilated_attn_bwd — the backward of the forward above: the gradients
 * of sum(dout * out) with respect to q, k and v.  The pages present LongNet
 * as a model that is trained ("LONGNET: Scaling Transformer to 1 billion
 * tokens", section "Distributed training"; "LongNet" docs page, features);
 * they give no formula for the gradient, so it is the exact derivative of the
 * forward's function.  Since the combination weighted by e^{lse_p} is one
 * softmax over all (pattern, key) pairs reaching a row, with
 * P_ij = e^{s_ij - lse_i}, delta_i = <dout_i, out_i> and
 * ds_ij = P_ij (<dout_i, v_j> - delta_i):
 *   dq_i = sum_j ds_ij k_j / sqrt(D), dk_j = sum_i ds_ij q_i / sqrt(D),
 *   dv_j = sum_i P_ij dout_i   (sums over the pairs of every pattern).
 *   - q, k, v, w, r, B, N, H, D, n_pat, causal, dtype: as given to the
 *     forward (same conventions).
 *   - out, lse: the forward's results for these inputs (device, out
 *     [B, N, H, D] in dtype, 16-byte aligned; lse fp32 [B, H, N], required,
 *     4-byte aligned).  lse is the combined one the forward writes.
 *   - dout: device [B, N, H, D] in dtype, the cotangent of out.
 *   - dq, dk, dv: device fp32 [B, N, H, D] (fp32 whatever dtype is, the
 *     precision gradients are accumulated in), 16-byte aligned, written in
 *     full (a row no pattern keeps gets zeros).  Must not alias the inputs.
 *   - flags: 0 or LONGNET_FLAG_QK_NORM, as given to the forward: the scores
 *     then use q / max(|q|, 1e-12) and k / max(|k|, 1e-12), and dq, dk are
 *     taken back through that normalisation (a (g - xhat <xhat, g>) per row,
 *     a = 1 / max(|x|, 1e-12); a g for a row with |x| <= 1e-12).  Other bits:
 *     LONGNET_ERR_INVALID_ARG.
 *   - impl: LONGNET_IMPL_AUTO (tcgen05 where it applies, else the tile
 *     kernels, else SIMT), LONGNET_IMPL_TCGEN05 (bf16/fp16, D = 16, 32, 64
 *     or 128, no qk_norm, up to 6 patterns: TMA-fed tcgen05 tensor cores with
 *     TMEM accumulators), LONGNET_IMPL_TILES (bf16/fp16, D = 64: mma.sync tensor
 *     cores) or LONGNET_IMPL_SIMT (fp32 FMA, D in {16, 32, 64, 128}, every
 *     dtype).  A family that does not cover the call: LONGNET_ERR_UNSUPPORTED.
 *   - Enqueued on stream; allocates nothing.  The tcgen05 and tile kernels
 *     zero dq, dk and dv on the stream first, then add each pattern's share
 *     with fp32 atomics, so the summation order of a row's patterns (at most
 *     n_pat terms) may vary between runs in the last bits; the tcgen05
 *     family also uses dq as scratch for delta before it computes dq.
 *     Returns a longnet_status.
 */
int longnet_dilated_attn_bwd(const void* q, const void* k, const void* v,
                             const void* out, const float* lse, const void* dout,
                             float* dq, float* dk, float* dv,
                             int64_t B, int64_t N, int64_t H, int64_t D,
                             int n_pat, const int64_t* w, const int64_t* r,
                             int causal, int dtype, int flags, int impl,
                             longnet_stream_t stream);

/*
 * longnet_dilated_attn_bwd_ws — the backward of longnet_dilated_attn_fwd_ws:
 * the gradients of sum(dout * out) with respect to the ORIGINAL q, k, v when
 * the forward applied the input-side options (flags: LONGNET_FLAG_QK_NORM,
 * LONGNET_FLAG_XPOS, or both; out and lse are that forward's results).  The
 * same prologue pass encodes q and k into the caller's workspace, the
 * attention's backward runs on the encoded rows (any family; AUTO picks as
 * for the plain backward, tcgen05 included), and a last pass takes dq and
 * dk back through XPOS (per element pair the transpose s R(-n theta_i), 1/s
 * for keys) and then the norm (a (g - xhat <xhat, g>)), in place.
 *   workspace, workspace_bytes: as for longnet_dilated_attn_fwd_ws (the
 *     encoded q and k are written there; contents on entry do not matter).
 *   flags = 0: the call is longnet_dilated_attn_bwd with flags 0 (workspace
 *     unused, may be null).  Other arguments, results and errors as
 *     longnet_dilated_attn_bwd and longnet_dilated_attn_fwd_ws.
 */
int longnet_dilated_attn_bwd_ws(const void* q, const void* k, const void* v,
                                const void* out, const float* lse, const void* dout,
                                float* dq, float* dk, float* dv,
                                int64_t B, int64_t N, int64_t H, int64_t D,
                                int n_pat, const int64_t* w, const int64_t* r,
                                int causal, int dtype, int flags, int impl,
                                void* workspace, int64_t workspace_bytes,
                                longnet_stream_t stream);

/*
 * longnet_select_impl — which family AUTO would run for these arguments
 * with lse requested (a longnet_impl >= 1), or a negative longnet_status
 * when the arguments are invalid.  Host-only; touches no device.  (Without
 * lse, a multi-pattern call the PATTERNS family would take goes to SIMT.)
 */
int longnet_select_impl(int64_t B, int64_t N, int64_t H, int64_t D, int n_pat,
                        const int64_t* w, const int64_t* r, int causal,
                        int dtype);

/*
 * longnet_last_device_status — synchronises `stream`, then returns and
 * clears the current device's status word: LONGNET_OK,
 * LONGNET_ERR_DEVICE_TIMEOUT when a kernel's bounded wait gave up (its
 * outputs are then undefined), or LONGNET_ERR_DEVICE_BOUNDS when a row index
 * given to longnet_gather_rows / longnet_scatter_rows was out of range (that
 * row was skipped; the attention kernels' index arithmetic is checked on the
 * host by the tests' walk restatements and carries no device-side check).
 * LONGNET_ERR_CUDA if the synchronisation itself failed.
 */
int longnet_last_device_status(longnet_stream_t stream);

/*
 * longnet_watchdog_selftest — enqueues one tiny kernel on `stream` that waits
 * on a shared-memory barrier nothing ever completes, with a wait limit of
 * `limit_ns` nanoseconds (clamped to [1e3, 1e9]).  The wait runs out, the
 * kernel records LONGNET_ERR_DEVICE_TIMEOUT in the status word and returns,
 * leaving the context usable.  Lets tests exercise the timeout path without
 * hanging a GPU.  Returns a longnet_status for the launch.
 */
int longnet_watchdog_selftest(int64_t limit_ns, longnet_stream_t stream);

/* Static text for a longnet_status code ("unknown status" otherwise). */
const char* longnet_status_string(int status);

/* Library version, e.g. "longnet-b200 1.0 sm_100a". */
const char* longnet_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LONGNET_H_ */
