/*
 * fa_oracle.c -- plain CPU reference for the exact attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header, table or helper with the
 * CUDA path.
 *
 * What it computes is the plain definition, row by row, in double precision:
 *
 *   O = softmax(scale * Q K^T + bias + mask) V,   LSE = log sum_j exp(score_j)
 *
 * following these passages of the source pages:
 *   - "mgoin/tml-fa4", argument contract: varlen layout q[total_q, Hq, D],
 *     k/v[total_k, Hkv, D], cu_seqlens int32 [B+1]; per-sequence lengths
 *     q_len_b = cu_q[b+1]-cu_q[b], k_len_b = cu_k[b+1]-cu_k[b]; the distance
 *     d = i + (k_len_b - q_len_b) - j; the bias term
 *     score[i, j, h] += rel_bias[cu_q[b] + i, h, d] when 0 <= d < rel_extent;
 *     and, in causal mode, d == 0 is the query's own key (so d < 0 is masked).
 *   - "flashrt/fa4-cute-runtime", forward_static: seqused_k gives the valid
 *     K/V length per batch entry of a padded buffer.
 *   - "flashrt/fa4-cute-runtime", Functions: the forward returns (out, lse).
 *   - "FlashAttention-4 backend for Blackwell #1235": the LSE lets a split over
 *     keys be combined outside the kernel (fa_oracle_lse_combine below).
 *
 * Readings where the pages are silent (each is listed with the design notes):
 *   - the bias is added after scaling and is itself unscaled;
 *   - query head h reads key/value head h / (Hq / Hkv);
 *   - with seqused_k, k_len_b = seqused_k[b] (also inside the distance rule),
 *     and keys are taken from the start of batch b's K/V rows;
 *   - the LSE is the natural logarithm;
 *   - a row with no admissible key gets O = 0 and LSE = -inf.
 *
 * Score and mask modifiers ("mgoin/tml-fa4" lists "mask/score modifiers"
 * among the forward paths without defining them; these are the plainest
 * readings, listed with the design notes):
 *   - sliding window: with d the distance above, a key is masked when
 *     d > window_left (too far left of the row's diagonal, window_left >= 0)
 *     or -d > window_right (too far right, window_right >= 0); a negative
 *     bound is no bound, and causal mode is window_right = 0;
 *   - soft-capping: with cap > 0 the scaled score s becomes cap * tanh(s / cap)
 *     before the bias is added.
 *
 * Inputs arrive as float arrays holding the exact bf16/fp16 input values
 * (both formats embed exactly in binary32); every product, sum, exponential
 * and logarithm below is done in double.
 *
 * No blocking, no online rescaling, no reordering: for each row the scores
 * are formed, their maximum taken, the exponentials summed, and O formed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Describes the packed problem.  Dense inputs are passed as varlen with
 * cu_q[b] = b*Sq and cu_k[b] = b*Sk. */
typedef struct {
  const float *q, *k, *v;       /* [total_q,Hq,D], [total_k,Hkv,D] x2 */
  const int *cu_q, *cu_k;       /* [B+1] */
  const int *seqused_k;         /* [B] or NULL */
  const float *rel_bias;        /* [total_q,Hq,R] or NULL */
  int B, Hq, Hkv, D, R, causal;
  double scale;
  int window_left, window_right; /* < 0: no bound */
  double softcap;                /* > 0: cap * tanh(s / cap); 0: off */
} fa_problem;

/* One attention row: batch b, query head h, query position i (0-based within
 * the sequence).  Keys are restricted to positions [kv_lo, kv_hi) of the
 * sequence (the whole sequence when kv_lo = 0, kv_hi = INT32_MAX); the split
 * form is what a split-KV partial computes.  Writes D outputs and the LSE.
 * Returns the number of admissible keys. */
static long attend_row(const fa_problem *p, int b, int h, int i, int kv_lo,
                       int kv_hi, double *o, double *lse, double *s_scratch) {
  const int G = p->Hq / p->Hkv;
  const int kvh = h / G;
  const int q_len = p->cu_q[b + 1] - p->cu_q[b];
  const int k_len = p->seqused_k ? p->seqused_k[b] : p->cu_k[b + 1] - p->cu_k[b];
  const long delta = (long)k_len - (long)q_len;
  const long qrow = (long)p->cu_q[b] + i;
  const float *qv = p->q + (qrow * p->Hq + h) * (long)p->D;
  const int D = p->D;

  int lo = kv_lo < 0 ? 0 : kv_lo;
  int hi = kv_hi > k_len ? k_len : kv_hi;

  /* scores of the admissible keys; -inf marks a masked key */
  double m = -INFINITY;
  long n_ok = 0;
  for (int j = lo; j < hi; ++j) {
    long d = (long)i + delta - (long)j;
    if ((p->causal && d < 0) || (p->window_left >= 0 && d > p->window_left) ||
        (p->window_right >= 0 && -d > p->window_right)) {
      s_scratch[j - lo] = -INFINITY;
      continue;
    }
    const float *kv = p->k + (((long)p->cu_k[b] + j) * p->Hkv + kvh) * (long)D;
    double acc = 0.0;
    for (int t = 0; t < D; ++t) acc += (double)qv[t] * (double)kv[t];
    double s = p->scale * acc;
    if (p->softcap > 0.0) s = p->softcap * tanh(s / p->softcap);
    if (p->rel_bias && d >= 0 && d < p->R)
      s += (double)p->rel_bias[(qrow * p->Hq + h) * (long)p->R + d];
    s_scratch[j - lo] = s;
    if (s > m) m = s;
    ++n_ok;
  }

  for (int t = 0; t < D; ++t) o[t] = 0.0;
  if (n_ok == 0 || m == -INFINITY) {
    *lse = -INFINITY;
    return n_ok;
  }
  double l = 0.0;
  for (int j = lo; j < hi; ++j) {
    double s = s_scratch[j - lo];
    if (s == -INFINITY) continue;
    double w = exp(s - m);
    l += w;
    const float *vv = p->v + (((long)p->cu_k[b] + j) * p->Hkv + kvh) * (long)D;
    for (int t = 0; t < D; ++t) o[t] += w * (double)vv[t];
  }
  for (int t = 0; t < D; ++t) o[t] /= l;
  *lse = m + log(l);
  return n_ok;
}

static int max_k_len(const fa_problem *p) {
  int mk = 0;
  for (int b = 0; b < p->B; ++b) {
    int kl = p->seqused_k ? p->seqused_k[b] : p->cu_k[b + 1] - p->cu_k[b];
    if (kl > mk) mk = kl;
  }
  return mk;
}

static int check_problem(const fa_problem *p) {
  if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->D <= 0) return 1;
  if (p->Hq % p->Hkv) return 2;
  if (p->rel_bias && p->R <= 0) return 3;
  if (!(p->softcap >= 0.0)) return 8;
  for (int b = 0; b < p->B; ++b) {
    if (p->cu_q[b + 1] < p->cu_q[b] || p->cu_k[b + 1] < p->cu_k[b]) return 4;
    if (p->seqused_k && (p->seqused_k[b] < 0 ||
                         p->seqused_k[b] > p->cu_k[b + 1] - p->cu_k[b]))
      return 5;
  }
  return 0;
}

/*
 * Every row of the problem.  out: [total_q, Hq, D] doubles; lse: [Hq, total_q]
 * doubles (the packed layout; callers reshape for dense).  The key window
 * [kv_lo, kv_hi) applies to every sequence (pass 0, INT32_MAX for all keys).
 * Returns 0 on success, a positive code on a malformed problem.
 */
int fa_oracle_forward(const float *q, const float *k, const float *v,
                      const int *cu_q, const int *cu_k, const int *seqused_k,
                      int B, int Hq, int Hkv, int D, int causal, double scale,
                      const float *rel_bias, int R, int kv_lo, int kv_hi,
                      double *out, double *lse, int nthreads, int window_left,
                      int window_right, double softcap) {
  fa_problem p = {q, k, v, cu_q, cu_k, seqused_k, rel_bias, B, Hq, Hkv, D, R,
                  causal, scale, window_left, window_right, softcap};
  int rc = check_problem(&p);
  if (rc) return rc;
  const long total_q = B > 0 ? cu_q[B] : 0;
  const int mk = max_k_len(&p);
  /* one work item = (packed query row, head) */
  const long items = total_q * Hq;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(mk > 0 ? mk : 1));
#pragma omp for schedule(dynamic, 16)
    for (long it = 0; it < items; ++it) {
      long row = it / Hq;
      int h = (int)(it % Hq);
      /* the sequence holding this packed row: cu_q[b] <= row < cu_q[b+1]
       * (binary search; empty sequences never hold a row) */
      int lo = 0, hi = B - 1;
      while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (cu_q[mid] <= row) lo = mid; else hi = mid - 1;
      }
      int b = lo;
      while (cu_q[b + 1] <= row) ++b;
      int i = (int)(row - cu_q[b]);
      attend_row(&p, b, h, i, kv_lo, kv_hi, out + (row * Hq + h) * (long)D,
                 lse + (long)h * total_q + row, s);
    }
    free(s);
  }
  return 0;
}

/*
 * A chosen list of rows (b, h, i), for problems too large to evaluate whole.
 * out: [n_rows, D] doubles, lse: [n_rows] doubles.
 */
int fa_oracle_rows(const float *q, const float *k, const float *v,
                   const int *cu_q, const int *cu_k, const int *seqused_k,
                   int B, int Hq, int Hkv, int D, int causal, double scale,
                   const float *rel_bias, int R, const int *row_b,
                   const int *row_h, const int *row_i, long n_rows,
                   double *out, double *lse, int nthreads, int window_left,
                   int window_right, double softcap) {
  fa_problem p = {q, k, v, cu_q, cu_k, seqused_k, rel_bias, B, Hq, Hkv, D, R,
                  causal, scale, window_left, window_right, softcap};
  int rc = check_problem(&p);
  if (rc) return rc;
  for (long r = 0; r < n_rows; ++r) {
    if (row_b[r] < 0 || row_b[r] >= B || row_h[r] < 0 || row_h[r] >= Hq)
      return 6;
    if (row_i[r] < 0 || row_i[r] >= cu_q[row_b[r] + 1] - cu_q[row_b[r]])
      return 7;
  }
  const int mk = max_k_len(&p);
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif
#pragma omp parallel
  {
    double *s = (double *)malloc(sizeof(double) * (size_t)(mk > 0 ? mk : 1));
#pragma omp for schedule(dynamic, 4)
    for (long r = 0; r < n_rows; ++r)
      attend_row(&p, row_b[r], row_h[r], row_i[r], 0, INT32_MAX,
                 out + r * (long)D, lse + r, s);
    free(s);
  }
  return 0;
}

/*
 * Merge of partial results over disjoint key ranges, as the TabPFN thread
 * describes doing split-KV outside the kernel with the returned LSE:
 *   lse = log sum_s exp(lse_s),  O = sum_s exp(lse_s - lse) * O_s.
 * Partials with lse_s = -inf carry no weight; if all are -inf, O = 0 and
 * lse = -inf.  o_parts: [n_splits, n_rows, D]; lse_parts: [n_splits, n_rows].
 */
void fa_oracle_lse_combine(const double *o_parts, const double *lse_parts,
                           int n_splits, long n_rows, int D, double *out,
                           double *lse) {
  for (long r = 0; r < n_rows; ++r) {
    double m = -INFINITY;
    for (int s = 0; s < n_splits; ++s)
      if (lse_parts[(long)s * n_rows + r] > m) m = lse_parts[(long)s * n_rows + r];
    double *o = out + r * (long)D;
    for (int t = 0; t < D; ++t) o[t] = 0.0;
    if (m == -INFINITY) {
      lse[r] = -INFINITY;
      continue;
    }
    double z = 0.0;
    for (int s = 0; s < n_splits; ++s) {
      double ls = lse_parts[(long)s * n_rows + r];
      if (ls == -INFINITY) continue;
      z += exp(ls - m);
    }
    double L = m + log(z);
    for (int s = 0; s < n_splits; ++s) {
      double ls = lse_parts[(long)s * n_rows + r];
      if (ls == -INFINITY) continue;
      double w = exp(ls - L);
      const double *os = o_parts + ((long)s * n_rows + r) * D;
      for (int t = 0; t < D; ++t) o[t] += w * os[t];
    }
    lse[r] = L;
  }
}

int fa_oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
