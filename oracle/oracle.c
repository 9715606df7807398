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
 *   6. the backward (oracle_dilated_attn_bwd_fp64 and its per-row form): the
 *      exact gradient of sum(dout * out) with respect to q, k and v, taking
 *      steps 5 to 1 in reverse; lse is not differentiated (it is saved for
 *      the backward).
 *
 * Layouts: q, k, v, out are [B, N, H, D] contiguous doubles; lse is [B, H, N]
 * (natural log, scale included).  Every pin against which this file is
 * checked lives in tests/oracle_pins.py (run by tests/test_oracle_pins.py;
 * tests/test_oracle_mutants.py runs them against planted mistakes).
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
 * Steps 1-4 for every pattern: the per-pattern outputs, materialised as
 * op [n_pat][B][N][H][D] and lp [n_pat][B][H][N] (allocated here, freed by
 * the caller).  Returns 0 or ORACLE_NO_MEMORY.
 */
static int forward_patterns(const double* q, const double* k, const double* v, int64_t B,
                            int64_t N, int64_t H, int64_t D, int n_pat, const int64_t* w,
                            const int64_t* r, int causal, double** op_out, double** lp_out) {
  const int64_t rows = B * N * H;
  double* op = (double*)malloc(sizeof(double) * (size_t)(n_pat * rows * D));
  double* lp = (double*)malloc(sizeof(double) * (size_t)(n_pat * rows));
  *op_out = op;
  *lp_out = lp;
  if (!op || !lp) return ORACLE_NO_MEMORY;
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
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
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
  double *op = NULL, *lp = NULL;
  rc = forward_patterns(q, k, v, B, N, H, D, n_pat, w, r, causal, &op, &lp);
  if (rc) {
    free(op);
    free(lp);
    return rc;
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
 * Pattern (wp, rp) for one row (b, pos, h): writes the row's attention output
 * over the kept rows of its segment into o (D doubles) and its lse into *l;
 * o = 0 and *l = -inf when the pattern does not keep the row.  sc is scratch
 * for min(wp, N) scores.
 */
static void row_pattern_attend(const double* q, const double* k, const double* v, int64_t N,
                               int64_t H, int64_t D, int64_t wp, int64_t rp, int causal,
                               int64_t b, int64_t pos, int64_t h, double* o, double* l,
                               double* sc) {
  const double scale = 1.0 / sqrt((double)D);
  const double* qi = q + ((b * N + pos) * H + h) * D;
  *l = -INFINITY;
  for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
  const int64_t seg = pos / wp;
  const int64_t o_h = h % rp;
  const int64_t off = pos - seg * wp - o_h;
  if (off < 0 || off % rp != 0) return; /* row not kept by this pattern */
  const int64_t i = off / rp;
  const int64_t m = rows_kept(seg_len(N, wp, seg), rp, o_h);
  const int64_t n_keys = causal ? i + 1 : m;
  double mx = -INFINITY;
  for (int64_t j = 0; j < n_keys; ++j) {
    const double* kj = k + ((b * N + seg * wp + o_h + rp * j) * H + h) * D;
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
    const double* vj = v + ((b * N + seg * wp + o_h + rp * j) * H + h) * D;
    for (int64_t d = 0; d < D; ++d) o[d] += sc[j] * vj[d];
  }
  for (int64_t d = 0; d < D; ++d) o[d] /= denom;
  *l = mx + log(denom);
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
        for (int p = 0; p < n_pat; ++p) {
          optr[p] = orows + p * D;
          row_pattern_attend(q, k, v, N, H, D, w[p], r[p], causal, b, pos, h, orows + p * D,
                             &lrow[p], sc);
        }
        combine_row(n_pat, lrow, optr, D, out_rows + t * D, lse_rows + t);
      }
    free(sc);
    free(orows);
  }
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/* ------------------------------------------------------------------------
 * Backward: the gradient of the forward above with respect to q, k and v.
 *
 * The pages present LongNet as a model one trains ("LongNet" docs page,
 * features list and training instructions; "LONGNET: Scaling Transformer to 1
 * billion tokens", section "Distributed training"), so the gradient of the
 * forward is the next step on the path.  The pages give no formula for it;
 * the reading adopted: the exact derivative of the function the forward
 * defines, differentiating the output `out` (lse is an auxiliary result that
 * is saved for the backward and receives no cotangent).  The steps are the
 * forward's, taken in reverse: step 5 (combination), then steps 4 to 1 per
 * (pattern, batch, head, segment), the scatter turning into a sum over the
 * patterns that keep a row.
 * ---------------------------------------------------------------------- */

/* Backward of combine_row.  With a_p = e^{lse_p - lse} the combination is
 * out = sum_p a_p O_p, and since lse = log sum_p e^{lse_p},
 * d out / d O_p = a_p and d out / d lse_p = a_p (O_p - out).  Given the
 * cotangent dout of the row it writes dO_p = a_p dout (D doubles at do_p[p])
 * and dlse_p = a_p <dout, O_p - out>; both are zero for patterns that do not
 * select the row. */
static void combine_row_bwd(int n_pat, const double* lse_p, const double* const* o_p,
                            const double* out, double lse, const double* dout, int64_t D,
                            double* const* do_p, double* dl_p) {
  for (int p = 0; p < n_pat; ++p) {
    if (lse_p[p] == -INFINITY) {
      for (int64_t d = 0; d < D; ++d) do_p[p][d] = 0.0;
      dl_p[p] = 0.0;
      continue;
    }
    const double a = exp(lse_p[p] - lse);
    double dot = 0.0;
    for (int64_t d = 0; d < D; ++d) {
      do_p[p][d] = a * dout[d];
      dot += dout[d] * (o_p[p][d] - out[d]);
    }
    dl_p[p] = a * dot;
  }
}

/* Backward of attend_segment on one sparsified segment.  With
 * p_ij = e^{s_ij - l_i}, o_i = sum_j p_ij v_j and l_i = log sum_j e^{s_ij}:
 * d o_i / d s_ij = p_ij (v_j - o_i) and d l_i / d s_ij = p_ij, so the score
 * cotangent is ds_ij = p_ij (<do_i, v_j> - <do_i, o_i> + dl_i); then
 * dv_j += p_ij do_i, dq_i += ds_ij k_j / sqrt(D), dk_j += ds_ij q_i / sqrt(D).
 * os and ls are the segment's outputs, dos and dls their cotangents; the
 * gradients are added into dqs, dks, dvs (m x D each). */
static void attend_segment_bwd(const double* qs, const double* ks, const double* vs,
                               const double* os, const double* ls, const double* dos,
                               const double* dls, double* dqs, double* dks, double* dvs,
                               int64_t m, int64_t D, int causal) {
  const double scale = 1.0 / sqrt((double)D);
  for (int64_t i = 0; i < m; ++i) {
    const int64_t n_keys = causal ? i + 1 : m;
    double delta = 0.0;
    for (int64_t d = 0; d < D; ++d) delta += dos[i * D + d] * os[i * D + d];
    for (int64_t j = 0; j < n_keys; ++j) {
      double s = 0.0, dp = 0.0;
      for (int64_t d = 0; d < D; ++d) {
        s += qs[i * D + d] * ks[j * D + d];
        dp += dos[i * D + d] * vs[j * D + d];
      }
      const double pij = exp(s * scale - ls[i]);
      const double ds = pij * (dp - delta + dls[i]);
      for (int64_t d = 0; d < D; ++d) {
        dvs[j * D + d] += pij * dos[i * D + d];
        dqs[i * D + d] += scale * ds * ks[j * D + d];
        dks[j * D + d] += scale * ds * qs[i * D + d];
      }
    }
  }
}

/*
 * Full backward.  q, k, v, dout are [B, N, H, D]; dq, dk, dv receive the
 * gradients of sum(dout * out) in the same layout.  The forward is recomputed
 * here (per-pattern outputs and the combination), so nothing from another
 * implementation enters.  Returns 0, or a negative code.
 */
int oracle_dilated_attn_bwd_fp64(const double* q, const double* k, const double* v,
                                 const double* dout, double* dq, double* dk, double* dv,
                                 int64_t B, int64_t N, int64_t H, int64_t D, int n_pat,
                                 const int64_t* w, const int64_t* r, int causal) {
  int rc = check_args(B, N, H, D, n_pat, w, r);
  if (rc) return rc;
  const int64_t rows = B * N * H;
  double *op = NULL, *lp = NULL;
  rc = forward_patterns(q, k, v, B, N, H, D, n_pat, w, r, causal, &op, &lp);
  double* dop = (double*)malloc(sizeof(double) * (size_t)(n_pat * rows * D));
  double* dlp = (double*)malloc(sizeof(double) * (size_t)(n_pat * rows));
  if (!rc && (!dop || !dlp)) rc = ORACLE_NO_MEMORY;
  if (rc) {
    free(op);
    free(lp);
    free(dop);
    free(dlp);
    return rc;
  }
  /* step 5 backwards: the combination's cotangents for every pattern */
#pragma omp parallel for schedule(static)
  for (int64_t row = 0; row < rows; ++row) {
    const int64_t h = row % H;
    const int64_t pos = (row / H) % N;
    const int64_t b = row / (H * N);
    double lrow[64], dlrow[64], out_row_lse;
    const double* orow[64];
    double* dorow[64];
    double out_row[1024];
    for (int p = 0; p < n_pat; ++p) {
      lrow[p] = lp[(int64_t)p * rows + (b * H + h) * N + pos];
      orow[p] = op + ((int64_t)p * rows + row) * D;
      dorow[p] = dop + ((int64_t)p * rows + row) * D;
    }
    double* outr = D <= 1024 ? out_row : (double*)malloc(sizeof(double) * (size_t)D);
    combine_row(n_pat, lrow, orow, D, outr, &out_row_lse);
    combine_row_bwd(n_pat, lrow, orow, outr, out_row_lse, dout + row * D, D, dorow, dlrow);
    for (int p = 0; p < n_pat; ++p) dlp[(int64_t)p * rows + (b * H + h) * N + pos] = dlrow[p];
    if (outr != out_row) free(outr);
  }
  memset(dq, 0, sizeof(double) * (size_t)(rows * D));
  memset(dk, 0, sizeof(double) * (size_t)(rows * D));
  memset(dv, 0, sizeof(double) * (size_t)(rows * D));
  /* steps 4..1 backwards, one pattern at a time: within a pattern the tasks
   * (batch, head, segment) own disjoint rows, so their sums do not collide */
  int failed = 0;
  for (int p = 0; p < n_pat && !failed; ++p) {
    const int64_t n_seg = (N + w[p] - 1) / w[p];
    const int64_t wcap = w[p] < N ? w[p] : N;
#pragma omp parallel
    {
      double* buf = (double*)malloc(sizeof(double) * (size_t)(wcap * (9 * D + 2)));
      const int have_buffers = buf != NULL;
#pragma omp for schedule(dynamic, 1)
      for (int64_t t = 0; t < B * H * n_seg; ++t) {
        if (!have_buffers) {
#pragma omp atomic write
          failed = 1;
          continue;
        }
        const int64_t seg = t % n_seg;
        const int64_t h = (t / n_seg) % H;
        const int64_t b = t / (n_seg * H);
        const int64_t o = h % r[p];
        const int64_t m = rows_kept(seg_len(N, w[p], seg), r[p], o);
        double *qs = buf, *ks = qs + wcap * D, *vs = ks + wcap * D, *os = vs + wcap * D;
        double *dos = os + wcap * D, *dqs = dos + wcap * D, *dks = dqs + wcap * D;
        double *dvs = dks + wcap * D, *ls = dvs + wcap * D, *dls = ls + wcap;
        for (int64_t i = 0; i < m; ++i) {
          const int64_t pos = seg * w[p] + o + r[p] * i;
          const int64_t row = (b * N + pos) * H + h;
          memcpy(qs + i * D, q + row * D, sizeof(double) * (size_t)D);
          memcpy(ks + i * D, k + row * D, sizeof(double) * (size_t)D);
          memcpy(vs + i * D, v + row * D, sizeof(double) * (size_t)D);
          memcpy(os + i * D, op + ((int64_t)p * rows + row) * D, sizeof(double) * (size_t)D);
          memcpy(dos + i * D, dop + ((int64_t)p * rows + row) * D, sizeof(double) * (size_t)D);
          ls[i] = lp[(int64_t)p * rows + (b * H + h) * N + pos];
          dls[i] = dlp[(int64_t)p * rows + (b * H + h) * N + pos];
        }
        memset(dqs, 0, sizeof(double) * (size_t)(3 * wcap * D));
        attend_segment_bwd(qs, ks, vs, os, ls, dos, dls, dqs, dks, dvs, m, D, causal);
        for (int64_t i = 0; i < m; ++i) {
          const int64_t row = (b * N + seg * w[p] + o + r[p] * i) * H + h;
          for (int64_t d = 0; d < D; ++d) {
            dq[row * D + d] += dqs[i * D + d];
            dk[row * D + d] += dks[i * D + d];
            dv[row * D + d] += dvs[i * D + d];
          }
        }
      }
      free(buf);
    }
  }
  free(op);
  free(lp);
  free(dop);
  free(dlp);
  return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/* Forward of one row over every pattern, then the combination's backward:
 * fills o_p (n_pat x D), l_p, the combined out (D) and lse, and the
 * cotangents do_p (n_pat x D) and dl_p that the row's dout gives each
 * pattern.  sc is scratch for min(max w, N) scores. */
static void row_cotangents(const double* q, const double* k, const double* v,
                           const double* dout, int64_t N, int64_t H, int64_t D, int n_pat,
                           const int64_t* w, const int64_t* r, int causal, int64_t b,
                           int64_t pos, int64_t h, double* o_p, double* l_p, double* out,
                           double* do_p, double* dl_p, double* sc) {
  const double* optr[64];
  double* doptr[64];
  double lse;
  for (int p = 0; p < n_pat; ++p) {
    optr[p] = o_p + p * D;
    doptr[p] = do_p + p * D;
    row_pattern_attend(q, k, v, N, H, D, w[p], r[p], causal, b, pos, h, o_p + p * D, &l_p[p],
                       sc);
  }
  combine_row(n_pat, l_p, optr, D, out, &lse);
  combine_row_bwd(n_pat, l_p, optr, out, lse, dout + ((b * N + pos) * H + h) * D, D, doptr,
                  dl_p);
}

/*
 * The backward for a list of single rows (b, pos, h), for sizes where the
 * full backward is too slow: dq of the row as a query, and dk, dv of the row
 * as a key, summing over every query that reaches it.  Each query's forward
 * and combination cotangents are recomputed from scratch.  rows_bph holds
 * n_rows triples; dq_rows, dk_rows, dv_rows are [n_rows][D].
 */
int oracle_dilated_attn_bwd_rows_fp64(const double* q, const double* k, const double* v,
                                      const double* dout, int64_t B, int64_t N, int64_t H,
                                      int64_t D, int n_pat, const int64_t* w, const int64_t* r,
                                      int causal, int64_t n_rows, const int64_t* rows_bph,
                                      double* dq_rows, double* dk_rows, double* dv_rows) {
  int rc = check_args(B, N, H, D, n_pat, w, r);
  if (rc) return rc;
  for (int64_t t = 0; t < n_rows; ++t) {
    const int64_t b = rows_bph[3 * t], pos = rows_bph[3 * t + 1], h = rows_bph[3 * t + 2];
    if (b < 0 || b >= B || pos < 0 || pos >= N || h < 0 || h >= H) return ORACLE_BAD_ARG;
  }
  const double scale = 1.0 / sqrt((double)D);
  int failed = 0;
#pragma omp parallel
  {
    int64_t wmax = 0;
    for (int p = 0; p < n_pat; ++p) wmax = w[p] > wmax ? w[p] : wmax;
    if (wmax > N) wmax = N;
    double* buf = (double*)malloc(sizeof(double) * (size_t)(wmax + n_pat * (4 * D + 2) + 2 * D));
    const int have_buffers = buf != NULL;
#pragma omp for schedule(dynamic, 1)
    for (int64_t t = 0; t < n_rows; ++t) {
      if (!have_buffers) {
#pragma omp atomic write
        failed = 1;
        continue;
      }
      double *sc = buf, *o_p = sc + wmax, *do_p = o_p + n_pat * D, *l_p = do_p + n_pat * D;
      double *dl_p = l_p + n_pat, *out = dl_p + n_pat, *o_p2 = out + D;
      double *do_p2 = o_p2 + n_pat * D, *out2 = do_p2 + n_pat * D;
      double l_p2[64], dl_p2[64];
      const int64_t b = rows_bph[3 * t], pos = rows_bph[3 * t + 1], h = rows_bph[3 * t + 2];
      double* dq_r = dq_rows + t * D;
      double* dk_r = dk_rows + t * D;
      double* dv_r = dv_rows + t * D;
      for (int64_t d = 0; d < D; ++d) dq_r[d] = dk_r[d] = dv_r[d] = 0.0;
      const double* qi = q + ((b * N + pos) * H + h) * D;
      const double* kr = k + ((b * N + pos) * H + h) * D;
      const double* vr = v + ((b * N + pos) * H + h) * D;
      /* the row as a query */
      row_cotangents(q, k, v, dout, N, H, D, n_pat, w, r, causal, b, pos, h, o_p, l_p, out, do_p,
                     dl_p, sc);
      for (int p = 0; p < n_pat; ++p) {
        if (l_p[p] == -INFINITY) continue;
        const int64_t seg = pos / w[p], o = h % r[p];
        const int64_t i = (pos - seg * w[p] - o) / r[p];
        const int64_t m = rows_kept(seg_len(N, w[p], seg), r[p], o);
        const int64_t n_keys = causal ? i + 1 : m;
        double delta = 0.0;
        for (int64_t d = 0; d < D; ++d) delta += do_p[p * D + d] * o_p[p * D + d];
        for (int64_t j = 0; j < n_keys; ++j) {
          const int64_t kp = seg * w[p] + o + r[p] * j;
          const double* kj = k + ((b * N + kp) * H + h) * D;
          const double* vj = v + ((b * N + kp) * H + h) * D;
          double s = 0.0, dp = 0.0;
          for (int64_t d = 0; d < D; ++d) {
            s += qi[d] * kj[d];
            dp += do_p[p * D + d] * vj[d];
          }
          const double pij = exp(s * scale - l_p[p]);
          const double ds = pij * (dp - delta + dl_p[p]);
          for (int64_t d = 0; d < D; ++d) dq_r[d] += scale * ds * kj[d];
        }
      }
      /* the row as a key: every query of the same sparsified segment that
       * attends to it (the ones at or after it when causal) */
      for (int p = 0; p < n_pat; ++p) {
        const int64_t seg = pos / w[p], o = h % r[p];
        const int64_t off = pos - seg * w[p] - o;
        if (off < 0 || off % r[p] != 0) continue; /* not a key of pattern p */
        const int64_t j = off / r[p];
        const int64_t m = rows_kept(seg_len(N, w[p], seg), r[p], o);
        for (int64_t i = causal ? j : 0; i < m; ++i) {
          const int64_t qp = seg * w[p] + o + r[p] * i;
          const double* qq = q + ((b * N + qp) * H + h) * D;
          row_cotangents(q, k, v, dout, N, H, D, n_pat, w, r, causal, b, qp, h, o_p2, l_p2, out2,
                         do_p2, dl_p2, sc);
          double s = 0.0, dp = 0.0, delta = 0.0;
          for (int64_t d = 0; d < D; ++d) {
            s += qq[d] * kr[d];
            dp += do_p2[p * D + d] * vr[d];
            delta += do_p2[p * D + d] * o_p2[p * D + d];
          }
          const double pij = exp(s * scale - l_p2[p]);
          const double ds = pij * (dp - delta + dl_p2[p]);
          for (int64_t d = 0; d < D; ++d) {
            dv_r[d] += pij * do_p2[p * D + d];
            dk_r[d] += scale * ds * qq[d];
          }
        }
      }
    }
    free(buf);
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
