/*
 * fp64 CPU oracle for the multi-pattern dilated-attention forward of LongNet.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the package's smoke check and the CPU
 * baseline leg of the benchmark use it.  It shares no code, header, table or
 * helper with the CUDA library; it is written from the method's description
 * alone, plainly and slowly, in double precision.
 *
 * What it computes, in the order the pages describe it:
 *   1. split the sequence into segments of w tokens; when w does not divide
 *      N the last segment is the shorter rest of the sequence (reading: no
 *      padding, the pages only speak of equal segments)
 *      ("LongNet论文精读", section "Dilated Attention的工作原理", first step;
 *       "LONGNET: Scaling Transformer to 1 billion tokens", section
 *       "LongNet's attention allocation principle");
 *   2. inside each segment keep every r-th row, head h starting at offset
 *      o = h mod r ("LONGNET: Scaling Transformer to 1 billion tokens",
 *      section "LongNet's attention allocation principle", the paragraph on
 *      heads having their own offset);
 *   3. run softmax attention with scale 1/sqrt(D) on each sparsified segment,
 *      causal inside the segment when asked ("LongNet论文精读", section
 *      "Dilated Attention的工作原理", third step);
 *   4. put the rows back at their positions (same section, fourth step);
 *   5. combine the patterns of the mixture ("LONGNET: Scaling Transformer to 1
 *      billion tokens", section "LongNet's attention allocation principle",
 *      the paragraph on a series of attention patterns; section "Token
 *      expansion reaches 1 billion+", combining local attention into global
 *      attention).  Reading adopted for the combination: each pattern's row is
 *      weighted by that pattern's softmax denominator exp(lse_p); rows a
 *      pattern does not select contribute nothing; a row no pattern selects
 *      gets out = 0 and lse = -inf.
 *
 * Layouts: q, k, v, out are [B, N, H, D] contiguous doubles; lse is [B, H, N]
 * (natural log, scale included).  Every pin against which this file is
 * checked lives in tests/test_oracle_pins.py.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG (-1)
#define ORACLE_NO_MEMORY (-2)

/* Number of rows head h keeps in one segment of pattern (w, r) whose length
 * is len (w, or less for a last segment cut by the end of the sequence): the
 * offsets o + r*k that stay below len. */
static int64_t rows_kept(int64_t len, int64_t r, int64_t o) {
  if (o >= len) return 0;
  return (len - o + r - 1) / r;
}

/* Length of segment seg of a pattern with segment length w: the sequence is
 * cut into segments of w tokens and the last one ends with the sequence. */
static int64_t seg_len(int64_t N, int64_t w, int64_t seg) {
  const int64_t rest = N - seg * w;
  return rest < w ? rest : w;
}

static int check_args(int64_t B, int64_t N, int64_t H, int64_t D, int n_pat,
                      const int64_t* w, const int64_t* r) {
  if (B <= 0 || N <= 0 || H <= 0 || D <= 0 || n_pat <= 0 || n_pat > 64) return ORACLE_BAD_ARG;
  for (int p = 0; p < n_pat; ++p) {
    if (r[p] < 1 || w[p] < 1) return ORACLE_BAD_ARG;
  }
  return ORACLE_OK;
}

/* Attention on one sparsified segment.  qs, ks, vs hold the m gathered rows
 * (m x D each).  For every query row i it writes the softmax-weighted sum of
 * value rows into os[i] and log(sum_j exp(s_ij)) into ls[i], where
 * s_ij = <q_i, k_j> / sqrt(D) and, when causal, only j <= i take part. */
static void attend_segment(const double* qs, const double* ks, const double* vs,
                           double* os, double* ls, int64_t m, int64_t D,
                           int causal, double* scores) {
  const double scale = 1.0 / sqrt((double)D);
  for (int64_t i = 0; i < m; ++i) {
    const int64_t n_keys = causal ? i + 1 : m;
    double mx = -INFINITY;
    for (int64_t j = 0; j < n_keys; ++j) {
      double s = 0.0;
      for (int64_t d = 0; d < D; ++d) s += qs[i * D + d] * ks[j * D + d];
      s *= scale;
      scores[j] = s;
      if (s > mx) mx = s;
    }
    double denom = 0.0;
    for (int64_t j = 0; j < n_keys; ++j) {
      scores[j] = exp(scores[j] - mx);
      denom += scores[j];
    }
    for (int64_t d = 0; d < D; ++d) {
      double acc = 0.0;
      for (int64_t j = 0; j < n_keys; ++j) acc += scores[j] * vs[j * D + d];
      os[i * D + d] = acc / denom;
    }
    ls[i] = mx + log(denom);
  }
}

/* Combine per-pattern results of one row: out = sum_p e^{lse_p} O_p / sum_p
 * e^{lse_p}, lse = log sum_p e^{lse_p}, over the patterns that selected the
 * row (finite lse_p).  The largest lse_p is taken out first. */
static void combine_row(int n_pat, const double* lse_p, const double* const* o_p,
                        int64_t D, double* out, double* lse) {
  double mx = -INFINITY;
  for (int p = 0; p < n_pat; ++p)
    if (lse_p[p] > mx) mx = lse_p[p];
  if (mx == -INFINITY) {
    for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
    *lse = -INFINITY;
    return;
  }
  double wsum = 0.0;
  for (int64_t d = 0; d < D; ++d) out[d] = 0.0;
  for (int p = 0; p < n_pat; ++p) {
    if (lse_p[p] == -INFINITY) continue;
    const double wt = exp(lse_p[p] - mx);
    wsum += wt;
    for (int64_t d = 0; d < D; ++d) out[d] += wt * o_p[p][d];
  }
  for (int64_t d = 0; d < D; ++d) out[d] /= wsum;
  *lse = mx + log(wsum);
}

/*
 * Full forward.  Per-pattern outputs are materialised ([n_pat][B][N][H][D]
 * and [n_pat][B][H][N]) and then combined row by row, exactly as the steps
 * above read.  Returns 0, or a negative code on bad arguments / no memory.
 */
int oracle_dilated_attn_fp64(const double* q, const double* k, const double* v,
                             double* out, double* lse, int64_t B, int64_t N,
                             int64_t H, int64_t D, int n_pat, const int64_t* w,
                             const int64_t* r, int causal) {
  int rc = check_args(B, N, H, D, n_pat, w, r);
  if (rc) return rc;
  const int64_t rows = B * N * H;
  double* op = (double*)malloc(sizeof(double) * (size_t)(n_pat * rows * D));
  double* lp = (double*)malloc(sizeof(double) * (size_t)(n_pat * rows));
  if (!op || !lp) {
    free(op);
    free(lp);
    return ORACLE_NO_MEMORY;
  }
  /* Rows a pattern does not select keep lse_p = -inf and O_p = 0. */
  for (int64_t i = 0; i < n_pat * rows; ++i) lp[i] = -INFINITY;
  memset(op, 0, sizeof(double) * (size_t)(n_pat * rows * D));

  /* One task per (pattern, batch, head, segment). */
  int64_t n_tasks_total = 0;
  int64_t task_base[64];
  for (int p = 0; p < n_pat; ++p) {
    task_base[p] = n_tasks_total;
    n_tasks_total += B * H * ((N + w[p] - 1) / w[p]);
  }
  int failed = 0;
#pragma omp parallel
  {
    int64_t wmax = 0;
    for (int p = 0; p < n_pat; ++p) wmax = w[p] > wmax ? w[p] : wmax;
    if (wmax > N) wmax = N; /* no segment is longer than the sequence */
    double* qs = (double*)malloc(sizeof(double) * (size_t)(wmax * D));
    double* ks = (double*)malloc(sizeof(double) * (size_t)(wmax * D));
    double* vs = (double*)malloc(sizeof(double) * (size_t)(wmax * D));
    double* os = (double*)malloc(sizeof(double) * (size_t)(wmax * D));
    double* ls = (double*)malloc(sizeof(double) * (size_t)wmax);
    double* sc = (double*)malloc(sizeof(double) * (size_t)wmax);
    const int have_buffers = qs && ks && vs && os && ls && sc;
    /* every thread reaches the work-sharing loop; a thread without buffers
     * only records the failure */
#pragma omp for schedule(dynamic, 1)
      for (int64_t t = 0; t < n_tasks_total; ++t) {
        if (!have_buffers) {
#pragma omp atomic write
          failed = 1;
          continue;
        }
        int p = 0;
        while (p + 1 < n_pat && t >= task_base[p + 1]) ++p;
        const int64_t n_seg = (N + w[p] - 1) / w[p];
        int64_t rem = t - task_base[p];
        const int64_t seg = rem % n_seg;
        rem /= n_seg;
        const int64_t h = rem % H;
        const int64_t b = rem / H;
        const int64_t o = h % r[p];
        const int64_t m = rows_kept(seg_len(N, w[p], seg), r[p], o);
        /* step 1+2: gather the kept rows of this segment */
        for (int64_t i = 0; i < m; ++i) {
          const int64_t pos = seg * w[p] + o + r[p] * i;
          const int64_t src = ((b * N + pos) * H + h) * D;
          memcpy(qs + i * D, q + src, sizeof(double) * (size_t)D);
          memcpy(ks + i * D, k + src, sizeof(double) * (size_t)D);
          memcpy(vs + i * D, v + src, sizeof(double) * (size_t)D);
        }
        /* step 3: dense attention on the sparsified segment */
        attend_segment(qs, ks, vs, os, ls, m, D, causal, sc);
        /* step 4: scatter back to the rows' positions */
        for (int64_t i = 0; i < m; ++i) {
          const int64_t pos = seg * w[p] + o + r[p] * i;
          const int64_t row = (b * N + pos) * H + h;
          memcpy(op + ((int64_t)p * rows + row) * D, os + i * D, sizeof(double) * (size_t)D);
          lp[(int64_t)p * rows + (b * H + h) * N + pos] = ls[i];
        }
      }
    free(qs);
    free(ks);
    free(vs);
    free(os);
    free(ls);
    free(sc);
  }
  if (failed) {
    free(op);
    free(lp);
    return ORACLE_NO_MEMORY;
  }
  /* step 5: combine the patterns row by row */
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < rows; ++row) {
    const int64_t h = row % H;
    const int64_t pos = (row / H) % N;
    const int64_t b = row / (H * N);
    double lrow[64];
    const double* orow[64];
    for (int p = 0; p < n_pat; ++p) {
      lrow[p] = lp[(int64_t)p * rows + (b * H + h) * N + pos];
      orow[p] = op + ((int64_t)p * rows + row) * D;
    }
    double l_out;
    combine_row(n_pat, lrow, orow, D, out + row * D, &l_out);
    if (lse) lse[(b * H + h) * N + pos] = l_out;
  }
  free(op);
  free(lp);
  return ORACLE_OK;
}

/*
 * The same forward for a list of single rows (b, pos, h), for sizes where the
 * full forward is too slow.  For every pattern that selects the row it gathers
 * that segment's kept key/value rows (up to the row itself when causal),
 * attends, and then combines the patterns as above.  rows_bph holds n_rows
 * triples; out_rows is [n_rows][D], lse_rows is [n_rows].
 */
int oracle_dilated_attn_rows_fp64(const double* q, const double* k, const double* v,
                                  int64_t B, int64_t N, int64_t H, int64_t D,
                                  int n_pat, const int64_t* w, const int64_t* r,
                                  int causal, int64_t n_rows, const int64_t* rows_bph,
                                  double* out_rows, double* lse_rows) {
  int rc = check_args(B, N, H, D, n_pat, w, r);
  if (rc) return rc;
  for (int64_t t = 0; t < n_rows; ++t) {
    const int64_t b = rows_bph[3 * t], pos = rows_bph[3 * t + 1], h = rows_bph[3 * t + 2];
    if (b < 0 || b >= B || pos < 0 || pos >= N || h < 0 || h >= H) return ORACLE_BAD_ARG;
  }
  int failed = 0;
#pragma omp parallel
  {
    int64_t wmax = 0;
    for (int p = 0; p < n_pat; ++p) wmax = w[p] > wmax ? w[p] : wmax;
    if (wmax > N) wmax = N; /* no segment is longer than the sequence */
    double* sc = (double*)malloc(sizeof(double) * (size_t)wmax);
    double* orows = (double*)malloc(sizeof(double) * (size_t)(64 * D));
    const int have_buffers = sc && orows;
    const double scale = 1.0 / sqrt((double)D);
#pragma omp for schedule(dynamic, 4)
      for (int64_t t = 0; t < n_rows; ++t) {
        if (!have_buffers) {
#pragma omp atomic write
          failed = 1;
          continue;
        }
        const int64_t b = rows_bph[3 * t], pos = rows_bph[3 * t + 1], h = rows_bph[3 * t + 2];
        double lrow[64];
        const double* optr[64];
        const double* qi = q + ((b * N + pos) * H + h) * D;
        for (int p = 0; p < n_pat; ++p) {
          double* oi = orows + p * D;
          optr[p] = oi;
          lrow[p] = -INFINITY;
          for (int64_t d = 0; d < D; ++d) oi[d] = 0.0;
          const int64_t seg = pos / w[p];
          const int64_t o = h % r[p];
          const int64_t off = pos - seg * w[p] - o;
          if (off < 0 || off % r[p] != 0) continue; /* row not kept by p */
          const int64_t i = off / r[p];
          const int64_t m = rows_kept(seg_len(N, w[p], seg), r[p], o);
          const int64_t n_keys = causal ? i + 1 : m;
          double mx = -INFINITY;
          for (int64_t j = 0; j < n_keys; ++j) {
            const double* kj = k + ((b * N + seg * w[p] + o + r[p] * j) * H + h) * D;
            double s = 0.0;
            for (int64_t d = 0; d < D; ++d) s += qi[d] * kj[d];
            s *= scale;
            sc[j] = s;
            if (s > mx) mx = s;
          }
          double denom = 0.0;
          for (int64_t j = 0; j < n_keys; ++j) {
            sc[j] = exp(sc[j] - mx);
            denom += sc[j];
          }
          for (int64_t j = 0; j < n_keys; ++j) {
            const double* vj = v + ((b * N + seg * w[p] + o + r[p] * j) * H + h) * D;
            for (int64_t d = 0; d < D; ++d) oi[d] += sc[j] * vj[d];
          }
          for (int64_t d = 0; d < D; ++d) oi[d] /= denom;
          lrow[p] = mx + log(denom);
        }
        combine_row(n_pat, lrow, optr, D, out_rows + t * D, lse_rows + t);
      }
    free(sc);
    free(orows);
  }
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/* Threads the OpenMP runtime will use (reported beside CPU timings). */
int oracle_num_threads(void) {
  int n = 1;
#pragma omp parallel
  {
#pragma omp single
    n = omp_get_num_threads();
  }
  return n;
}
