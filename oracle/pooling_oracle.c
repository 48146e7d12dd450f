/*
 * Seed-query attention pooling oracle: plain, slow, fp64 CPU implementation
 * of the first level of Hierarchical Seed Pooling.  TEST INFRASTRUCTURE ONLY:
 * the tests call it; the product library never does, and this file shares no
 * code, header or constant with it.
 *
 * What it computes.  The Kunlun summary (gist.science, "Resumen Tecnico:
 * Kunlun", section 2.2, HSP bullet) says HSP replaces the random learnable
 * queries of PMA (pooling by multi-head attention) with learned seed-level
 * representations for long sequences, before a SumKronLinear compression; the
 * RecSysChannel review (item 3) places it after GDPA.  The first level is
 * read (R21) as PMA's attention with learned seeds: per head j, S seed
 * queries attend over the n_b tokens of sample b:
 *
 *   Q^ = seeds[j] (S x dh),  K^ = K[off[b]:off[b+1], j, :],  V^ likewise (n_b x dh)
 *   A  = s Q^ K^T (S x n_b),  P = row softmax(A),  O[b, j] = P V^ (S x dh)
 *   LSE[b, j, i] = M_i + ln sum_t exp(A_it - M_i),  M_i = max_t A_it
 *
 * A sample without tokens pools nothing: O = 0 and LSE = -inf (reading).
 * Gradient for an upstream dO [B, h, S, dh]:
 *
 *   dV^ = P^T dO^,  dP = dO^ V^T,  dA = P * (dP - D),  D_i = sum_t P_it dP_it,
 *   dK^ = s dA^T Q^,  dseeds[j] = s sum_b dA_b K^_b   (the seeds are shared).
 *
 * Every sum is a plain loop in double; units (b, j) run under OpenMP and the
 * seed gradient is summed over samples afterwards in sample order.
 * Layouts: seeds, dseeds [h, S, dh]; k, v, dk, dv [T, h, dh] (jagged, int64
 * offsets [B+1]); o, dout [B, h, S, dh]; lse [B, h, S].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int valid(int B, int h, int dh, int S, const int64_t* off) {
  if (B < 0 || h <= 0 || dh <= 0 || S <= 0 || !off || off[0] != 0) return 0;
  for (int b = 0; b < B; ++b)
    if (off[b + 1] < off[b]) return 0;
  return 1;
}

/* P (S x n) = row softmax of s Q^ K^T for one unit; LSE per row. */
static void probs(int S, int n, int dh, int h, const float* qb, const float* kb, double scale,
                  double* P, double* lse) {
  for (int i = 0; i < S; ++i) {
    double mx = -INFINITY;
    for (int t = 0; t < n; ++t) {
      double acc = 0.0;
      for (int d = 0; d < dh; ++d) acc += (double)qb[(size_t)i * dh + d] * (double)kb[(size_t)t * h * dh + d];
      P[(size_t)i * n + t] = scale * acc;
      mx = P[(size_t)i * n + t] > mx ? P[(size_t)i * n + t] : mx;
    }
    double sum = 0.0;
    for (int t = 0; t < n; ++t) sum += exp(P[(size_t)i * n + t] - mx);
    for (int t = 0; t < n; ++t) P[(size_t)i * n + t] = exp(P[(size_t)i * n + t] - mx) / sum;
    if (lse) lse[i] = mx + log(sum);
  }
}

int pool_oracle_fwd(int B, int h, int dh, int S, const int64_t* off, const float* seeds,
                    const float* k, const float* v, double scale, double* o, double* lse,
                    int nthreads) {
  if (!valid(B, h, dh, S, off) || !seeds || !k || !v || !o) return -1;
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (long u = 0; u < (long)B * h; ++u) {
    const int b = (int)(u / h), j = (int)(u % h);
    const int n = (int)(off[b + 1] - off[b]);
    double* ob = o + (size_t)u * S * dh;
    double* lb = lse ? lse + (size_t)u * S : NULL;
    if (n == 0) {
      memset(ob, 0, sizeof(double) * (size_t)S * dh);
      if (lb)
        for (int i = 0; i < S; ++i) lb[i] = -INFINITY;
      continue;
    }
    double* P = (double*)malloc(sizeof(double) * (size_t)S * n);
    if (!P) {
      failed |= 1;
      continue;
    }
    const float* qb = seeds + (size_t)j * S * dh;
    const float* kb = k + ((size_t)off[b] * h + j) * dh;
    const float* vb = v + ((size_t)off[b] * h + j) * dh;
    probs(S, n, dh, h, qb, kb, scale, P, lb);
    for (int i = 0; i < S; ++i)
      for (int d = 0; d < dh; ++d) {
        double acc = 0.0;
        for (int t = 0; t < n; ++t) acc += P[(size_t)i * n + t] * (double)vb[(size_t)t * h * dh + d];
        ob[(size_t)i * dh + d] = acc;
      }
    free(P);
  }
  return failed ? -2 : 0;
}

int pool_oracle_bwd(int B, int h, int dh, int S, const int64_t* off, const float* seeds,
                    const float* k, const float* v, const float* dout, double scale,
                    double* dseeds, double* dk, double* dv, int nthreads) {
  if (!valid(B, h, dh, S, off) || !seeds || !k || !v || !dout || !dseeds || !dk || !dv) return -1;
  const int64_t T = off[B];
  memset(dk, 0, sizeof(double) * (size_t)T * h * dh);
  memset(dv, 0, sizeof(double) * (size_t)T * h * dh);
  double* dq_units = (double*)calloc((size_t)B * h * S * dh, sizeof(double));
  if (!dq_units && (size_t)B * h * S * dh > 0) return -2;
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (long u = 0; u < (long)B * h; ++u) {
    const int b = (int)(u / h), j = (int)(u % h);
    const int n = (int)(off[b + 1] - off[b]);
    if (n == 0) continue;
    double* P = (double*)malloc(sizeof(double) * (size_t)S * n);
    double* dA = (double*)malloc(sizeof(double) * (size_t)S * n);
    if (!P || !dA) {
      free(P); free(dA);
      failed |= 1;
      continue;
    }
    const float* qb = seeds + (size_t)j * S * dh;
    const float* kb = k + ((size_t)off[b] * h + j) * dh;
    const float* vb = v + ((size_t)off[b] * h + j) * dh;
    const float* gb = dout + (size_t)u * S * dh;
    double* dkb = dk + ((size_t)off[b] * h + j) * dh;
    double* dvb = dv + ((size_t)off[b] * h + j) * dh;
    probs(S, n, dh, h, qb, kb, scale, P, NULL);
    /* dP = dO V^T, then dA = P * (dP - D) in place */
    for (int i = 0; i < S; ++i) {
      double D = 0.0;
      for (int t = 0; t < n; ++t) {
        double acc = 0.0;
        for (int d = 0; d < dh; ++d) acc += (double)gb[(size_t)i * dh + d] * (double)vb[(size_t)t * h * dh + d];
        dA[(size_t)i * n + t] = acc;
        D += P[(size_t)i * n + t] * acc;
      }
      for (int t = 0; t < n; ++t) dA[(size_t)i * n + t] = P[(size_t)i * n + t] * (dA[(size_t)i * n + t] - D);
    }
    /* dV^ = P^T dO^, dK^ = s dA^T Q^ */
    for (int t = 0; t < n; ++t)
      for (int d = 0; d < dh; ++d) {
        double av = 0.0, ak = 0.0;
        for (int i = 0; i < S; ++i) {
          av += P[(size_t)i * n + t] * (double)gb[(size_t)i * dh + d];
          ak += dA[(size_t)i * n + t] * (double)qb[(size_t)i * dh + d];
        }
        dvb[(size_t)t * h * dh + d] = av;
        dkb[(size_t)t * h * dh + d] = scale * ak;
      }
    /* this unit's share of the seed gradient: s dA K^ */
    double* dqu = dq_units + (size_t)u * S * dh;
    for (int i = 0; i < S; ++i)
      for (int d = 0; d < dh; ++d) {
        double acc = 0.0;
        for (int t = 0; t < n; ++t) acc += dA[(size_t)i * n + t] * (double)kb[(size_t)t * h * dh + d];
        dqu[(size_t)i * dh + d] = scale * acc;
      }
    free(P); free(dA);
  }
  /* dseeds[j] = sum over samples, in sample order */
  for (int j = 0; j < h; ++j)
    for (size_t e = 0; e < (size_t)S * dh; ++e) {
      double acc = 0.0;
      for (int b = 0; b < B; ++b) acc += dq_units[((size_t)b * h + j) * S * dh + e];
      dseeds[(size_t)j * S * dh + e] = acc;
    }
  free(dq_units);
  return failed ? -2 : 0;
}
