/*
 * oracle.c -- plain, slow, fp64 CPU oracle for SPAttention band-sparse attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this code.  The product path (the
 * CUDA library and its Python binding) never calls it and shares no code,
 * header, table or helper with it.
 *
 * Sources ("Making Every Head Count: Sparse Attention Without the
 * Speed-Performance Trade-off", arXiv 2511.09596, and the blog post
 * "Story of Attention -- Part 4: Sparse Attention, Then and Now"):
 *
 *   - Balanced Distance Partitioning: the causal distance range [0, N) is cut
 *     into H contiguous, non-overlapping bands of width floor(N/H) or
 *     ceil(N/H); head 0 takes the nearest band, head H-1 the farthest
 *     ("Making Every Head Count", Figure 1 caption; abstract).  The pages give
 *     the widths but no formula; the bands used here are
 *     lo_h = floor(h*N/H), hi_h = floor((h+1)*N/H).
 *   - Sparse attention keeps the attention formula and only restricts the set
 *     of keys that the softmax runs over ("Story of Attention -- Part 4",
 *     section 1, the Sparse-Attention equation and the remark after it):
 *         o_i = sum_{j in S_i} exp(s_ij) / sum_{m in S_i} exp(s_im) * v_j,
 *         s_ij = scale * q_i . k_j.
 *   - For SPAttention, S_i^h = { j : 0 <= j <= i, lo_h <= i - j < hi_h }.
 *   - A row whose permitted set is empty (i < lo_h) outputs o_i = 0 and
 *     lse_i = -inf (a convention; the pages are silent on it).
 *   - The pages never write the backward pass.  It is the gradient of the
 *     forward above, derived by hand: with L = sum(O * dO),
 *         P_ij  = exp(s_ij - lse_i)            (j in S_i),
 *         D_i   = sum_c dO_ic * o_ic,
 *         dP_ij = dO_i . v_j,
 *         dS_ij = P_ij * (dP_ij - D_i),
 *         dq_i  = scale * sum_j dS_ij k_j,
 *         dk_j  = scale * sum_i dS_ij q_i,
 *         dv_j  = sum_i P_ij dO_i.
 *
 * Every permitted set is enumerated explicitly, row by row, in double
 * precision.  There is no tiling, no online softmax and no reordering beyond
 * the sums written above.  OpenMP only splits independent rows or heads
 * across threads.
 *
 * Tensor layout: [B][H][N][d] contiguous doubles; lse is [B][H][N].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Balanced Distance Partitioning (Figure 1 caption of "Making Every Head    */
/* Count"): band of head h is [lo[h], hi[h]).  Returns 0, or -1 on bad args. */
/* ------------------------------------------------------------------------ */
int oracle_bands(int64_t N, int64_t H, int64_t* lo, int64_t* hi) {
  if (N < 1 || H < 1 || H > N) return -1;
  for (int64_t h = 0; h < H; ++h) {
    lo[h] = (h * N) / H;
    hi[h] = ((h + 1) * N) / H;
  }
  return 0;
}

/* Is key j permitted for query i under band [lo, hi)?  (causal, 0 <= j <= i) */
static int permitted(int64_t i, int64_t j, int64_t lo, int64_t hi) {
  if (j < 0 || j > i) return 0;
  return (i - j >= lo) && (i - j < hi);
}

/* Number of permitted (i, j) pairs of one head over a length-N sequence,
 * counted one pair at a time. */
int64_t oracle_band_pairs(int64_t N, int64_t lo, int64_t hi) {
  int64_t count = 0;
  for (int64_t i = 0; i < N; ++i)
    for (int64_t j = 0; j <= i; ++j)
      count += permitted(i, j, lo, hi);
  return count;
}

static double dot(const double* a, const double* b, int64_t d) {
  double s = 0.0;
  for (int64_t c = 0; c < d; ++c) s += a[c] * b[c];
  return s;
}

/* ------------------------------------------------------------------------ */
/* Generic masked softmax attention on one head ("Story of Attention --      */
/* Part 4", section 1, Sparse-Attention equation).  mask[i*nk + j] != 0      */
/* means key j is in S_i.  Outputs:                                          */
/*   scores[nq*nk] (may be NULL): scale*q_i.k_j for every pair (unmasked),   */
/*   attn[nq*nk]   (may be NULL): softmax weights, 0 outside S_i,            */
/*   o[nq*d], lse[nq].  Empty S_i gives o_i = 0, lse_i = -inf.               */
/* ------------------------------------------------------------------------ */
void oracle_masked_attn_fwd(const double* q, const double* k, const double* v,
                            const uint8_t* mask, int64_t nq, int64_t nk, int64_t d,
                            double scale, double* scores, double* attn,
                            double* o, double* lse) {
  double* s = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
  for (int64_t i = 0; i < nq; ++i) {
    double m = -INFINITY;
    int64_t count = 0;
    for (int64_t j = 0; j < nk; ++j) {
      s[j] = scale * dot(q + i * d, k + j * d, d);
      if (scores) scores[i * nk + j] = s[j];
      if (mask[i * nk + j]) {
        if (s[j] > m) m = s[j];
        ++count;
      }
    }
    for (int64_t c = 0; c < d; ++c) o[i * d + c] = 0.0;
    if (count == 0) {
      lse[i] = -INFINITY;
      if (attn)
        for (int64_t j = 0; j < nk; ++j) attn[i * nk + j] = 0.0;
      continue;
    }
    double l = 0.0;
    for (int64_t j = 0; j < nk; ++j)
      if (mask[i * nk + j]) l += exp(s[j] - m);
    lse[i] = m + log(l);
    for (int64_t j = 0; j < nk; ++j) {
      double p = mask[i * nk + j] ? exp(s[j] - lse[i]) : 0.0;
      if (attn) attn[i * nk + j] = p;
      if (p != 0.0)
        for (int64_t c = 0; c < d; ++c) o[i * d + c] += p * v[j * d + c];
    }
  }
  free(s);
}

/* Gradient of L = sum(O * dout) for the generic masked attention above. */
void oracle_masked_attn_bwd(const double* q, const double* k, const double* v,
                            const uint8_t* mask, int64_t nq, int64_t nk, int64_t d,
                            double scale, const double* dout,
                            double* dq, double* dk, double* dv) {
  double* o = (double*)calloc((size_t)(nq * d), sizeof(double));
  double* lse = (double*)calloc((size_t)nq, sizeof(double));
  oracle_masked_attn_fwd(q, k, v, mask, nq, nk, d, scale, NULL, NULL, o, lse);
  memset(dq, 0, sizeof(double) * (size_t)(nq * d));
  memset(dk, 0, sizeof(double) * (size_t)(nk * d));
  memset(dv, 0, sizeof(double) * (size_t)(nk * d));
  for (int64_t i = 0; i < nq; ++i) {
    if (isinf(lse[i])) continue; /* empty S_i: the row contributes nothing */
    double Di = dot(dout + i * d, o + i * d, d);
    for (int64_t j = 0; j < nk; ++j) {
      if (!mask[i * nk + j]) continue;
      double sij = scale * dot(q + i * d, k + j * d, d);
      double p = exp(sij - lse[i]);
      double dp = dot(dout + i * d, v + j * d, d);
      double ds = p * (dp - Di);
      for (int64_t c = 0; c < d; ++c) {
        dq[i * d + c] += scale * ds * k[j * d + c];
        dk[j * d + c] += scale * ds * q[i * d + c];
        dv[j * d + c] += p * dout[i * d + c];
      }
    }
  }
  free(o);
  free(lse);
}

/* ------------------------------------------------------------------------ */
/* SPAttention forward of one row: head slices qh, kh, vh are [N][d].        */
/* S_i = { j : max(0, i-hi+1) <= j <= i-lo }, enumerated explicitly.         */
/* Writes o_i[d]; returns lse_i (natural log), -inf when S_i is empty.       */
/* ------------------------------------------------------------------------ */
static double spa_row_fwd(const double* qh, const double* kh, const double* vh,
                          int64_t N, int64_t d, double scale, int64_t lo, int64_t hi,
                          int64_t i, double* o_i) {
  (void)N;
  for (int64_t c = 0; c < d; ++c) o_i[c] = 0.0;
  int64_t jlo = i - hi + 1;
  if (jlo < 0) jlo = 0;
  int64_t jhi = i - lo;
  if (jhi < jlo) return -INFINITY;
  double m = -INFINITY;
  for (int64_t j = jlo; j <= jhi; ++j) {
    double s = scale * dot(qh + i * d, kh + j * d, d);
    if (s > m) m = s;
  }
  double l = 0.0;
  for (int64_t j = jlo; j <= jhi; ++j)
    l += exp(scale * dot(qh + i * d, kh + j * d, d) - m);
  double lse = m + log(l);
  for (int64_t j = jlo; j <= jhi; ++j) {
    double p = exp(scale * dot(qh + i * d, kh + j * d, d) - lse);
    for (int64_t c = 0; c < d; ++c) o_i[c] += p * vh[j * d + c];
  }
  return lse;
}

/* Forward for a list of flat row ids r = (b*H + h)*N + i.  o_rows[nrows][d],
 * lse_rows[nrows].  lo/hi give each head's band. */
void oracle_spa_fwd_rows(const double* q, const double* k, const double* v,
                         int64_t B, int64_t H, int64_t N, int64_t d, double scale,
                         const int64_t* lo, const int64_t* hi,
                         const int64_t* rows, int64_t nrows,
                         double* o_rows, double* lse_rows) {
  (void)B;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t flat = rows[r];
    int64_t bh = flat / N, i = flat % N, h = bh % H;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    lse_rows[r] = spa_row_fwd(qh, kh, vh, N, d, scale, lo[h], hi[h], i, o_rows + r * d);
  }
}

/* Forward over the whole tensor. */
void oracle_spa_fwd(const double* q, const double* k, const double* v,
                    int64_t B, int64_t H, int64_t N, int64_t d, double scale,
                    const int64_t* lo, const int64_t* hi, double* o, double* lse) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t flat = 0; flat < B * H * N; ++flat) {
    int64_t bh = flat / N, i = flat % N, h = bh % H;
    lse[flat] = spa_row_fwd(q + bh * N * d, k + bh * N * d, v + bh * N * d, N, d, scale,
                            lo[h], hi[h], i, o + flat * d);
  }
}

/* ------------------------------------------------------------------------ */
/* Backward over the whole tensor: gradients of L = sum(O * dout).           */
/* One (b, h) slice per task, so dk/dv accumulation never races.             */
/* ------------------------------------------------------------------------ */
void oracle_spa_bwd(const double* q, const double* k, const double* v, const double* dout,
                    int64_t B, int64_t H, int64_t N, int64_t d, double scale,
                    const int64_t* lo, const int64_t* hi,
                    double* dq, double* dk, double* dv) {
  memset(dq, 0, sizeof(double) * (size_t)(B * H * N * d));
  memset(dk, 0, sizeof(double) * (size_t)(B * H * N * d));
  memset(dv, 0, sizeof(double) * (size_t)(B * H * N * d));
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < B * H; ++bh) {
    int64_t h = bh % H;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    const double* doh = dout + bh * N * d;
    double* dqh = dq + bh * N * d;
    double* dkh = dk + bh * N * d;
    double* dvh = dv + bh * N * d;
    double* o_i = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t i = 0; i < N; ++i) {
      double lse = spa_row_fwd(qh, kh, vh, N, d, scale, lo[h], hi[h], i, o_i);
      if (isinf(lse)) continue; /* empty band row: no gradient flows */
      double Di = dot(doh + i * d, o_i, d);
      int64_t jlo = i - hi[h] + 1;
      if (jlo < 0) jlo = 0;
      int64_t jhi = i - lo[h];
      for (int64_t j = jlo; j <= jhi; ++j) {
        double s = scale * dot(qh + i * d, kh + j * d, d);
        double p = exp(s - lse);
        double dp = dot(doh + i * d, vh + j * d, d);
        double ds = p * (dp - Di);
        for (int64_t c = 0; c < d; ++c) {
          dqh[i * d + c] += scale * ds * kh[j * d + c];
          dkh[j * d + c] += scale * ds * qh[i * d + c];
          dvh[j * d + c] += p * doh[i * d + c];
        }
      }
    }
    free(o_i);
  }
}

/* ------------------------------------------------------------------------ */
/* Exclusive bands plus a local window shared by every head: a reading of   */
/* Figure 2(b) of "Making Every Head Count", whose EBALL ablation takes     */
/* local sharing out.  The pages never define the shared part;              */
/* here head h attends to S_i = { j <= i : i - j < w  or  lo_h <= i - j <   */
/* hi_h }, enumerated one key at a time.  w = 0 is the plain band.          */
/* ------------------------------------------------------------------------ */
static int union_permitted(int64_t i, int64_t j, int64_t w, int64_t lo, int64_t hi) {
  if (j < 0 || j > i) return 0;
  return (i - j < w) || ((i - j >= lo) && (i - j < hi));
}

static double union_row_fwd(const double* qh, const double* kh, const double* vh,
                            int64_t d, double scale, int64_t w, int64_t lo, int64_t hi,
                            int64_t i, double* o_i) {
  for (int64_t c = 0; c < d; ++c) o_i[c] = 0.0;
  double m = -INFINITY;
  int64_t count = 0;
  for (int64_t j = 0; j <= i; ++j) {
    if (!union_permitted(i, j, w, lo, hi)) continue;
    double s = scale * dot(qh + i * d, kh + j * d, d);
    if (s > m) m = s;
    ++count;
  }
  if (count == 0) return -INFINITY;
  double l = 0.0;
  for (int64_t j = 0; j <= i; ++j)
    if (union_permitted(i, j, w, lo, hi)) l += exp(scale * dot(qh + i * d, kh + j * d, d) - m);
  double lse = m + log(l);
  for (int64_t j = 0; j <= i; ++j) {
    if (!union_permitted(i, j, w, lo, hi)) continue;
    double p = exp(scale * dot(qh + i * d, kh + j * d, d) - lse);
    for (int64_t c = 0; c < d; ++c) o_i[c] += p * vh[j * d + c];
  }
  return lse;
}

void oracle_union_fwd(const double* q, const double* k, const double* v,
                      int64_t B, int64_t H, int64_t N, int64_t d, double scale, int64_t w,
                      const int64_t* lo, const int64_t* hi, double* o, double* lse) {
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t flat = 0; flat < B * H * N; ++flat) {
    int64_t bh = flat / N, i = flat % N, h = bh % H;
    lse[flat] = union_row_fwd(q + bh * N * d, k + bh * N * d, v + bh * N * d, d, scale, w,
                              lo[h], hi[h], i, o + flat * d);
  }
}

void oracle_union_fwd_rows(const double* q, const double* k, const double* v,
                           int64_t B, int64_t H, int64_t N, int64_t d, double scale, int64_t w,
                           const int64_t* lo, const int64_t* hi, const int64_t* rows,
                           int64_t nrows, double* o_rows, double* lse_rows) {
  (void)B;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t flat = rows[r];
    int64_t bh = flat / N, i = flat % N, h = bh % H;
    lse_rows[r] = union_row_fwd(q + bh * N * d, k + bh * N * d, v + bh * N * d, d, scale, w,
                                lo[h], hi[h], i, o_rows + r * d);
  }
}

/* Gradients of L = sum(O * dout) for the union above (same derivation as
 * oracle_spa_bwd, over the union's permitted set). */
void oracle_union_bwd(const double* q, const double* k, const double* v, const double* dout,
                      int64_t B, int64_t H, int64_t N, int64_t d, double scale, int64_t w,
                      const int64_t* lo, const int64_t* hi, double* dq, double* dk, double* dv) {
  memset(dq, 0, sizeof(double) * (size_t)(B * H * N * d));
  memset(dk, 0, sizeof(double) * (size_t)(B * H * N * d));
  memset(dv, 0, sizeof(double) * (size_t)(B * H * N * d));
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t bh = 0; bh < B * H; ++bh) {
    int64_t h = bh % H;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    const double* doh = dout + bh * N * d;
    double* dqh = dq + bh * N * d;
    double* dkh = dk + bh * N * d;
    double* dvh = dv + bh * N * d;
    double* o_i = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t i = 0; i < N; ++i) {
      double lse = union_row_fwd(qh, kh, vh, d, scale, w, lo[h], hi[h], i, o_i);
      if (isinf(lse)) continue;
      double Di = dot(doh + i * d, o_i, d);
      for (int64_t j = 0; j <= i; ++j) {
        if (!union_permitted(i, j, w, lo[h], hi[h])) continue;
        double s = scale * dot(qh + i * d, kh + j * d, d);
        double p = exp(s - lse);
        double dp = dot(doh + i * d, vh + j * d, d);
        double ds = p * (dp - Di);
        for (int64_t c = 0; c < d; ++c) {
          dqh[i * d + c] += scale * ds * kh[j * d + c];
          dkh[j * d + c] += scale * ds * qh[i * d + c];
          dvh[j * d + c] += p * doh[i * d + c];
        }
      }
    }
    free(o_i);
  }
}

/* dQ of the union for a list of query rows (flat ids as in oracle_spa_fwd_rows). */
void oracle_union_bwd_dq_rows(const double* q, const double* k, const double* v,
                              const double* dout, int64_t B, int64_t H, int64_t N, int64_t d,
                              double scale, int64_t w, const int64_t* lo, const int64_t* hi,
                              const int64_t* rows, int64_t nrows, double* dq_rows) {
  (void)B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t flat = rows[r];
    int64_t bh = flat / N, i = flat % N, h = bh % H;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    const double* doh = dout + bh * N * d;
    double* out = dq_rows + r * d;
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    double* o_i = (double*)malloc(sizeof(double) * (size_t)d);
    double lse = union_row_fwd(qh, kh, vh, d, scale, w, lo[h], hi[h], i, o_i);
    if (!isinf(lse)) {
      double Di = dot(doh + i * d, o_i, d);
      for (int64_t j = 0; j <= i; ++j) {
        if (!union_permitted(i, j, w, lo[h], hi[h])) continue;
        double p = exp(scale * dot(qh + i * d, kh + j * d, d) - lse);
        double ds = p * (dot(doh + i * d, vh + j * d, d) - Di);
        for (int64_t c = 0; c < d; ++c) out[c] += scale * ds * kh[j * d + c];
      }
    }
    free(o_i);
  }
}

/* dK and dV of the union for a list of key rows r = (b*H + h)*N + j: every
 * query i >= j whose set holds key j, its forward row recomputed first. */
void oracle_union_bwd_dkdv_rows(const double* q, const double* k, const double* v,
                                const double* dout, int64_t B, int64_t H, int64_t N, int64_t d,
                                double scale, int64_t w, const int64_t* lo, const int64_t* hi,
                                const int64_t* rows, int64_t nrows, double* dk_rows,
                                double* dv_rows) {
  (void)B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t flat = rows[r];
    int64_t bh = flat / N, j = flat % N, h = bh % H;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    const double* doh = dout + bh * N * d;
    double* dkr = dk_rows + r * d;
    double* dvr = dv_rows + r * d;
    for (int64_t c = 0; c < d; ++c) dkr[c] = dvr[c] = 0.0;
    double* o_i = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t i = j; i < N; ++i) {
      if (!union_permitted(i, j, w, lo[h], hi[h])) continue;
      double lse = union_row_fwd(qh, kh, vh, d, scale, w, lo[h], hi[h], i, o_i);
      double Di = dot(doh + i * d, o_i, d);
      double p = exp(scale * dot(qh + i * d, kh + j * d, d) - lse);
      double ds = p * (dot(doh + i * d, vh + j * d, d) - Di);
      for (int64_t c = 0; c < d; ++c) {
        dkr[c] += scale * ds * qh[i * d + c];
        dvr[c] += p * doh[i * d + c];
      }
    }
    free(o_i);
  }
}

/* dQ for a list of query rows (flat ids as in oracle_spa_fwd_rows). */
void oracle_spa_bwd_dq_rows(const double* q, const double* k, const double* v,
                            const double* dout, int64_t B, int64_t H, int64_t N, int64_t d,
                            double scale, const int64_t* lo, const int64_t* hi,
                            const int64_t* rows, int64_t nrows, double* dq_rows) {
  (void)B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t flat = rows[r];
    int64_t bh = flat / N, i = flat % N, h = bh % H;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    const double* doh = dout + bh * N * d;
    double* out = dq_rows + r * d;
    for (int64_t c = 0; c < d; ++c) out[c] = 0.0;
    double* o_i = (double*)malloc(sizeof(double) * (size_t)d);
    double lse = spa_row_fwd(qh, kh, vh, N, d, scale, lo[h], hi[h], i, o_i);
    if (!isinf(lse)) {
      double Di = dot(doh + i * d, o_i, d);
      int64_t jlo = i - hi[h] + 1;
      if (jlo < 0) jlo = 0;
      for (int64_t j = jlo; j <= i - lo[h]; ++j) {
        double p = exp(scale * dot(qh + i * d, kh + j * d, d) - lse);
        double ds = p * (dot(doh + i * d, vh + j * d, d) - Di);
        for (int64_t c = 0; c < d; ++c) out[c] += scale * ds * kh[j * d + c];
      }
    }
    free(o_i);
  }
}

/* dK and dV for a list of key rows r = (b*H + h)*N + j.  Every query i that
 * reaches key j (j + lo <= i <= min(j + hi - 1, N - 1)) has its own forward
 * row recomputed first. */
void oracle_spa_bwd_dkdv_rows(const double* q, const double* k, const double* v,
                              const double* dout, int64_t B, int64_t H, int64_t N, int64_t d,
                              double scale, const int64_t* lo, const int64_t* hi,
                              const int64_t* rows, int64_t nrows,
                              double* dk_rows, double* dv_rows) {
  (void)B;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < nrows; ++r) {
    int64_t flat = rows[r];
    int64_t bh = flat / N, j = flat % N, h = bh % H;
    const double* qh = q + bh * N * d;
    const double* kh = k + bh * N * d;
    const double* vh = v + bh * N * d;
    const double* doh = dout + bh * N * d;
    double* dkr = dk_rows + r * d;
    double* dvr = dv_rows + r * d;
    for (int64_t c = 0; c < d; ++c) dkr[c] = dvr[c] = 0.0;
    double* o_i = (double*)malloc(sizeof(double) * (size_t)d);
    int64_t ihi = j + hi[h] - 1;
    if (ihi > N - 1) ihi = N - 1;
    for (int64_t i = j + lo[h]; i <= ihi; ++i) {
      double lse = spa_row_fwd(qh, kh, vh, N, d, scale, lo[h], hi[h], i, o_i);
      double Di = dot(doh + i * d, o_i, d);
      double p = exp(scale * dot(qh + i * d, kh + j * d, d) - lse);
      double ds = p * (dot(doh + i * d, vh + j * d, d) - Di);
      for (int64_t c = 0; c < d; ++c) {
        dkr[c] += scale * ds * qh[i * d + c];
        dvr[c] += p * doh[i * d + c];
      }
    }
    free(o_i);
  }
}

/* ------------------------------------------------------------------------ */
/* Tile classes by brute force.  A (query tile t, key tile u) of size        */
/* Bq x Bk covers rows [t*Bq, t*Bq+Bq) and keys [u*Bk, u*Bk+Bk).  Positions  */
/* at or past N count as not permitted.  cls[(h*nqt + t)*nkt + u] =          */
/*   0 when no element of the tile is permitted,                             */
/*   2 when every element is permitted,                                      */
/*   1 otherwise.                                                            */
/* ------------------------------------------------------------------------ */
void oracle_tile_classes(int64_t N, int64_t H, const int64_t* lo, const int64_t* hi,
                         int64_t Bq, int64_t Bk, uint8_t* cls) {
  int64_t nqt = (N + Bq - 1) / Bq, nkt = (N + Bk - 1) / Bk;
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
  for (int64_t h = 0; h < H; ++h) {
    for (int64_t t = 0; t < nqt; ++t) {
      for (int64_t u = 0; u < nkt; ++u) {
        int64_t allowed = 0;
        for (int64_t i = t * Bq; i < t * Bq + Bq; ++i)
          for (int64_t j = u * Bk; j < u * Bk + Bk; ++j)
            allowed += (i < N && j < N && permitted(i, j, lo[h], hi[h]));
        cls[(h * nqt + t) * nkt + u] = allowed == 0 ? 0 : (allowed == Bq * Bk ? 2 : 1);
      }
    }
  }
}
