/*
 * entmax_oracle.c -- plain fp64 CPU oracle for causal alpha-entmax attention (forward pass).
 *
 * TEST INFRASTRUCTURE.  Only the test-suite, the smoke check and the CPU-baseline leg of the
 * benchmark load this file.  It shares no code, header, table or helper with the CUDA library,
 * and the library never calls it.
 *
 * What is computed, per attention head h and query row i (AdaSplash: Adaptive Sparse Flash
 * Attention, sections "AdaSplash with Block Masking", "Adaptive Sparsity Control",
 * "Variable Length Sequences" and "Causal and Non-causal Masking"; the closed form of
 * alpha-entmax is the one of Peters, Niculae & Martins 2019, "Sparse Sequence-to-Sequence
 * Models", which those pages build on but do not print):
 *
 *   s_ij = q_i . k_j / sqrt(d)          k, v taken from kv head floor(h / (Hq / Hkv))
 *   z_ij = (alpha - 1) s_ij
 *   p_ij = [z_ij - tau_i]_+ ^ (1 / (alpha - 1)),   tau_i the unique value with sum_j p_ij = 1
 *   o_i  = sum_j p_ij v_j                  (no renormalisation)
 *
 * over the valid keys j: j <= i inside the row's own sequence when causal, the whole sequence
 * otherwise.  The block mask of the "AdaSplash with Block Masking" section has one bit per
 * (128-row query tile, 128-key key tile); this file reports, per row and key tile, the largest
 * p of the row inside the tile, from which the tile bit is "any p > 0" by definition.
 *
 * tau is found exactly (up to fp64 rounding), not by a fixed number of iterations:
 *   1. tau >= m - 1 where m = max_j z_ij, because p_ij <= 1; so only keys with z > m - 1 can be
 *      in the support ("candidates").
 *   2. Sort the candidates descending: z_(1) >= z_(2) >= ...  The support size k* is the largest
 *      r with F(z_(r)) = sum_{t<r} (z_(t) - z_(r))^beta < 1 (F is nondecreasing in r).
 *   3. On the support, solve sum_{t<=k*} (z_(t) - tau)^beta = 1 on
 *      [max(z_(k*+1), m - 1), z_(k*)):
 *        beta = 1 (alpha = 2, sparsemax): tau = (sum z - 1) / k*
 *        beta = 2 (alpha = 1.5):          tau = mean - sqrt(1/k* - var)
 *        otherwise: safeguarded Newton inside the interval, run until it stops moving.
 *
 * oracle_tau_halley() separately writes out the fixed-iteration bracketed Halley + bisection
 * search named in the "Triton Entmax (Optimized Entmax Activation)" section, in fp64, so the
 * tests can check how far n_iter steps of that search get on a given input.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_TILE 128 /* query-tile and key-tile edge of the block mask */

/* ------------------------------------------------------------------------------------------ */
/* Row-level alpha-entmax.                                                                     */
/* ------------------------------------------------------------------------------------------ */

static int cmp_desc(const void* a, const void* b) {
  double x = *(const double*)a, y = *(const double*)b;
  return (x < y) - (x > y);
}

/* (z_t - tau)^beta summed over the first k entries of a descending list, and its derivative
 * with respect to tau. */
static void support_sums(const double* zs, int k, double tau, double beta, double* g, double* dg) {
  double s0 = 0.0, s1 = 0.0;
  for (int t = 0; t < k; ++t) {
    double x = zs[t] - tau;
    if (x > 0.0) {
      s0 += pow(x, beta);
      s1 += pow(x, beta - 1.0);
    }
  }
  *g = s0 - 1.0;
  *dg = -beta * s1;
}

/* Exact tau from the sorted (descending) candidates zs[0..nc) of a row with maximum m.
 * force_general = 1 skips the closed forms and always runs the safeguarded solver. */
static double tau_from_sorted(const double* zs, int nc, double m, double beta, int force_general) {
  /* Step 2: support size.  F(z_(1)) = 0 < 1, so k* >= 1. */
  int ks = 1;
  for (int r = 2; r <= nc; ++r) {
    double F = 0.0;
    for (int t = 0; t < r - 1; ++t) F += pow(zs[t] - zs[r - 1], beta);
    if (F < 1.0) ks = r;
    else break; /* F is nondecreasing in r */
  }
  double lo = (ks < nc) ? zs[ks] : m - 1.0;
  if (lo < m - 1.0) lo = m - 1.0;
  double hi = zs[ks - 1];

  if (!force_general && beta == 1.0) {
    double sum = 0.0;
    for (int t = 0; t < ks; ++t) sum += zs[t];
    return (sum - 1.0) / ks;
  }
  if (!force_general && beta == 2.0) {
    double mean = 0.0;
    for (int t = 0; t < ks; ++t) mean += zs[t];
    mean /= ks;
    double var = 0.0;
    for (int t = 0; t < ks; ++t) var += (zs[t] - mean) * (zs[t] - mean);
    var /= ks;
    double rad = 1.0 / ks - var;
    if (rad < 0.0) rad = 0.0; /* only reachable through rounding */
    return mean - sqrt(rad);
  }

  /* Safeguarded Newton on g(tau) = sum_{t<=k*} (z_t - tau)^beta - 1, convex and decreasing on
   * [lo, hi] with g(lo) >= 0 > g(hi): from lo the Newton iterates rise monotonically to the
   * root; the bracket guards against rounding. */
  double tau = lo;
  for (int it = 0; it < 200; ++it) {
    double g, dg;
    support_sums(zs, ks, tau, beta, &g, &dg);
    if (g == 0.0) return tau;
    if (g > 0.0) lo = tau;
    else hi = tau;
    double nt = (dg < 0.0) ? tau - g / dg : 0.5 * (lo + hi);
    if (!(nt > lo && nt < hi)) nt = 0.5 * (lo + hi);
    double tol = 2.0 * DBL_EPSILON * fmax(1.0, fabs(tau));
    if (fabs(nt - tau) <= tol || hi - lo <= 2.0 * tol) return nt;
    tau = nt;
  }
  return tau;
}

/* tau of the vector z[0..n), n >= 1.  work must hold n doubles. */
static double tau_of_vector(const double* z, int n, double alpha, int force_general, double* work) {
  double beta = 1.0 / (alpha - 1.0);
  double m = -INFINITY;
  for (int j = 0; j < n; ++j)
    if (z[j] > m) m = z[j];
  int nc = 0;
  for (int j = 0; j < n; ++j)
    if (z[j] > m - 1.0) work[nc++] = z[j];
  qsort(work, (size_t)nc, sizeof(double), cmp_desc);
  return tau_from_sorted(work, nc, m, beta, force_general);
}

/* Exported: tau and p of one vector (alpha-entmax of z). */
int oracle_entmax_vec(const double* z, int n, double alpha, int force_general, double* p_out,
                      double* tau_out) {
  if (n < 1 || !(alpha > 1.0)) return 1;
  double* work = (double*)malloc(sizeof(double) * (size_t)n);
  if (!work) return 2;
  double tau = tau_of_vector(z, n, alpha, force_general, work);
  free(work);
  double beta = 1.0 / (alpha - 1.0);
  if (p_out)
    for (int j = 0; j < n; ++j) p_out[j] = (z[j] > tau) ? pow(z[j] - tau, beta) : 0.0;
  if (tau_out) *tau_out = tau;
  return 0;
}

/* Exported: the fixed-iteration bracketed Halley + bisection search for tau, in fp64.
 * Start tau = m - 1 with bracket [m - 1, m - n^(1 - alpha)].  Each of the n_iter steps
 * evaluates f = sum [z - tau]_+^beta - 1 and its first two derivatives and narrows the bracket
 * by the sign of f.  It proposes the Halley step tau - 2 f f' / (2 f'^2 - f f'') when that
 * denominator is positive and finite (the step then points at the root), else the Newton step
 * - f / f'.  The proposal is taken if it lies in the closed bracket [lo, hi] and either is
 * within rounding of tau or is at most half as long as the step before last (the progress test
 * of the safeguarded Newton method "rtsafe", Press et al., Numerical Recipes); otherwise the
 * bracket midpoint is taken.  The closed bracket keeps a converged tau in place; the progress
 * test breaks the two-cycles that the infinite slope of [z - tau]_+^beta at a support edge
 * causes when beta < 1.  Returns the last tau. */
double oracle_tau_halley(const double* z, int n, double alpha, int n_iter) {
  double beta = 1.0 / (alpha - 1.0);
  double m = -INFINITY;
  for (int j = 0; j < n; ++j)
    if (z[j] > m) m = z[j];
  double lo = m - 1.0;
  double hi = m - pow((double)n, 1.0 - alpha);
  double tau = lo;
  double dx = hi - lo, dxold = hi - lo; /* the last two step lengths */
  for (int it = 0; it < n_iter; ++it) {
    double s0 = 0.0, s1 = 0.0, s2 = 0.0;
    for (int j = 0; j < n; ++j) {
      double x = z[j] - tau;
      if (x > 0.0) {
        s0 += pow(x, beta);
        s1 += pow(x, beta - 1.0);
        if (beta != 1.0) s2 += pow(x, beta - 2.0);
      }
    }
    double f = s0 - 1.0;
    double f1 = -beta * s1;
    double f2 = (beta != 1.0) ? beta * (beta - 1.0) * s2 : 0.0;
    if (f > 0.0) lo = tau;
    else hi = tau;
    double den = 2.0 * f1 * f1 - f * f2;
    double nt = (den > 0.0 && isfinite(den)) ? tau - 2.0 * f * f1 / den : tau - f / f1;
    double step = fabs(nt - tau);
    int small = step <= 4.0 * DBL_EPSILON * fmax(1.0, fabs(tau));
    if (!isfinite(nt) || !(nt >= lo && nt <= hi) || !(small || step <= 0.5 * dxold))
      nt = 0.5 * (lo + hi);
    dxold = dx;
    dx = fabs(nt - tau);
    tau = nt;
  }
  return tau;
}

/* ------------------------------------------------------------------------------------------ */
/* Attention rows.                                                                             */
/* ------------------------------------------------------------------------------------------ */

/* Layout (the heads-before-tokens layout of the "AdaSplash with Block Masking" example):
 *   fixed length: q [B, Hq, T, d], k and v [B, Hkv, T, d]; row id r = (b * Hq + h) * T + t
 *   varlen (cu_seqlens != NULL, nseq sequences packed back to back, T = total tokens):
 *                 q [Hq, T, d], k and v [Hkv, T, d]; row id r = h * T + t, t a packed position
 * All arrays hold fp32 values; bf16 tensors are widened by the caller (an exact conversion).
 *
 * For each of the nrows requested rows:
 *   tau_out[i]                  exact tau (or tau_given[i] when tau_given != NULL)
 *   o_out[i * d + c]            o_i, when o_out != NULL
 *   maxp[i * maxp_stride + kt]  max of p_ij over the valid keys j of key tile kt, counted from
 *                               the start of the row's sequence; 0 where the row has no valid
 *                               key; when maxp != NULL.  maxp_stride >= number of key tiles.
 * With tau_given, p is evaluated at that tau instead of the exact one (used to decide mask
 * bits that sit within rounding of the threshold).
 * Returns 0, or 1 on a malformed argument.                                                    */
int oracle_entmax_attn_rows(const float* q, const float* k, const float* v, int B, int Hq, int Hkv,
                            int T, int d, double alpha, int causal, const int32_t* cu_seqlens,
                            int nseq, const int64_t* rows, int64_t nrows, const double* tau_given,
                            double* tau_out, double* o_out, double* maxp, int64_t maxp_stride,
                            int nthreads) {
  if (B < 1 || Hq < 1 || Hkv < 1 || T < 1 || d < 1 || Hq % Hkv != 0 || !(alpha > 1.0)) return 1;
  if (cu_seqlens && (nseq < 1 || cu_seqlens[0] != 0 || cu_seqlens[nseq] != T)) return 1;
  const int G = Hq / Hkv;
  const double scale = 1.0 / sqrt((double)d);
  const double beta = 1.0 / (alpha - 1.0);
  const int64_t nrow_total = cu_seqlens ? (int64_t)Hq * T : (int64_t)B * Hq * T;
  for (int64_t i = 0; i < nrows; ++i)
    if (rows[i] < 0 || rows[i] >= nrow_total) return 1;
  if (maxp) { /* every key tile of the longest sequence needs a slot */
    int64_t longest = T;
    if (cu_seqlens) {
      longest = 0;
      for (int b = 0; b < nseq; ++b)
        if (cu_seqlens[b + 1] - cu_seqlens[b] > longest) longest = cu_seqlens[b + 1] - cu_seqlens[b];
    }
    if (maxp_stride < (longest + ORACLE_TILE - 1) / ORACLE_TILE) return 1;
  }
  int err = 0;

#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#else
  (void)nthreads;
#endif

#pragma omp parallel
  {
    double* z = (double*)malloc(sizeof(double) * (size_t)T);
    double* work = (double*)malloc(sizeof(double) * (size_t)T);
    double* qd = (double*)malloc(sizeof(double) * (size_t)d);
    double* od = (double*)malloc(sizeof(double) * (size_t)d);
    if (!z || !work || !qd || !od) {
#pragma omp atomic write
      err = 2;
    } else {
#pragma omp for schedule(dynamic, 4)
      for (int64_t ii = 0; ii < nrows; ++ii) {
        int64_t r = rows[ii];
        int b, h, t;       /* batch, q head, token position (packed for varlen) */
        int64_t seq0, len; /* first token of the row's sequence and its length */
        const float *qrow, *kbase, *vbase;
        if (cu_seqlens) {
          h = (int)(r / T);
          t = (int)(r % T);
          b = 0;
          while (b + 1 < nseq && cu_seqlens[b + 1] <= t) ++b;
          seq0 = cu_seqlens[b];
          len = cu_seqlens[b + 1] - cu_seqlens[b];
          qrow = q + ((int64_t)h * T + t) * d;
          kbase = k + (int64_t)(h / G) * T * d;
          vbase = v + (int64_t)(h / G) * T * d;
        } else {
          t = (int)(r % T);
          h = (int)((r / T) % Hq);
          b = (int)(r / ((int64_t)T * Hq));
          seq0 = 0;
          len = T;
          qrow = q + r * d;
          kbase = k + ((int64_t)b * Hkv + h / G) * T * d;
          vbase = v + ((int64_t)b * Hkv + h / G) * T * d;
        }
        int64_t pos = t - seq0; /* position inside the sequence */
        int64_t j_end = causal ? pos + 1 : len; /* valid keys: seq0 + [0, j_end) */
        int n = (int)j_end;

        for (int c = 0; c < d; ++c) qd[c] = (double)qrow[c];
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) {
          const float* kj = kbase + (seq0 + j) * d;
          double dot = 0.0;
          /* the simd reduction only lets the compiler split the sum into partial sums */
#pragma omp simd reduction(+ : dot)
          for (int c = 0; c < d; ++c) dot += qd[c] * (double)kj[c];
          double s = dot * scale;
          z[j] = (alpha - 1.0) * s;
          if (z[j] > m) m = z[j];
        }

        double tau;
        if (tau_given) {
          tau = tau_given[ii];
        } else {
          int nc = 0;
          for (int j = 0; j < n; ++j)
            if (z[j] > m - 1.0) work[nc++] = z[j];
          qsort(work, (size_t)nc, sizeof(double), cmp_desc);
          tau = tau_from_sorted(work, nc, m, beta, 0);
        }
        tau_out[ii] = tau;

        if (o_out)
          for (int c = 0; c < d; ++c) od[c] = 0.0;
        if (maxp)
          for (int64_t kt = 0; kt < maxp_stride; ++kt) maxp[ii * maxp_stride + kt] = 0.0;
        for (int j = 0; j < n; ++j) {
          if (!(z[j] > tau)) continue;
          double p = pow(z[j] - tau, beta);
          if (o_out) {
            const float* vj = vbase + (seq0 + j) * d;
            for (int c = 0; c < d; ++c) od[c] += p * (double)vj[c];
          }
          if (maxp) {
            double* slot = &maxp[ii * maxp_stride + j / ORACLE_TILE];
            if (p > *slot) *slot = p;
          }
        }
        if (o_out)
          for (int c = 0; c < d; ++c) o_out[ii * d + c] = od[c];
      }
    }
    free(z);
    free(work);
    free(qd);
    free(od);
  }
  return err;
}

/* Exported: number of OpenMP threads a parallel region would use (1 without OpenMP). */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
