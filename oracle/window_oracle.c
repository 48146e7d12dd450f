/*
 * Sliding-window self-attention oracle: plain, slow, fp64 CPU implementation
 * of attention restricted to a local window of each sample's jagged token
 * sequence.  TEST INFRASTRUCTURE ONLY: the tests call it; the product library
 * never does, and this file shares no code, header or constant with it.
 *
 * What it computes.  The Kunlun summary (gist.science, "Resumen Tecnico:
 * Kunlun", section 2.2, sliding-window bullet) says that self-attention on the
 * sequence is restricted to local windows, taking its cost from O(T^2) to
 * O(T w); the page gives neither the window's alignment nor its width.  The
 * reading taken (R22) is the causal window of width w: token t of a sample
 * attends to the tokens t' of the same sample with t - w < t' <= t.  Per
 * sample b and head j, with rows of Q, K, V [T, h, dh]:
 *
 *   A_tt' = s q_t . k_t'   for t - w < t' <= t, t' in the sample
 *   O_t   = sum_t' softmax_t'(A_t.) v_t',   LSE_t = ln sum_t' exp(A_tt')
 *
 * (every token sees at least itself, so no row is empty).  Gradient for dO:
 *
 *   dV_t' = sum_t P_tt' dO_t,  dP_tt' = dO_t . v_t',  dA = P * (dP - D_t),
 *   D_t = sum_t' P_tt' dP_tt',  dQ_t = s sum_t' dA_tt' k_t',  dK_t' = s sum_t dA_tt' q_t.
 *
 * Every sum is a plain loop in double over the window; units (b, j) run under
 * OpenMP.  Layouts: q, k, v, o, dout, dq, dk, dv [T, h, dh]; lse [h, T];
 * offsets int64 [B+1].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int valid(int B, int h, int dh, int w, const int64_t* off) {
  if (B < 0 || h <= 0 || dh <= 0 || w <= 0 || !off || off[0] != 0) return 0;
  for (int b = 0; b < B; ++b)
    if (off[b + 1] < off[b]) return 0;
  return 1;
}

static double dot(const float* a, const float* b, int dh) {
  double acc = 0.0;
  for (int d = 0; d < dh; ++d) acc += (double)a[d] * (double)b[d];
  return acc;
}

/* The window of token t (sample start t0): t' in [lo, t]. */
static int64_t window_lo(int64_t t, int64_t t0, int w) {
  const int64_t lo = t - w + 1;
  return lo > t0 ? lo : t0;
}

int win_oracle_fwd(int B, int h, int dh, int w, const int64_t* off, const float* q,
                   const float* k, const float* v, double scale, double* o, double* lse,
                   int nthreads) {
  if (!valid(B, h, dh, w, off) || !q || !k || !v || !o) return -1;
  const int64_t T = off[B];
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1)
  for (long u = 0; u < (long)B * h; ++u) {
    const int b = (int)(u / h), j = (int)(u % h);
    for (int64_t t = off[b]; t < off[b + 1]; ++t) {
      const int64_t lo = window_lo(t, off[b], w);
      const float* qt = q + ((size_t)t * h + j) * dh;
      double mx = -INFINITY;
      for (int64_t s = lo; s <= t; ++s) {
        const double a = scale * dot(qt, k + ((size_t)s * h + j) * dh, dh);
        mx = a > mx ? a : mx;
      }
      double sum = 0.0;
      double* ot = o + ((size_t)t * h + j) * dh;
      for (int d = 0; d < dh; ++d) ot[d] = 0.0;
      for (int64_t s = lo; s <= t; ++s) {
        const double p = exp(scale * dot(qt, k + ((size_t)s * h + j) * dh, dh) - mx);
        sum += p;
        const float* vs = v + ((size_t)s * h + j) * dh;
        for (int d = 0; d < dh; ++d) ot[d] += p * (double)vs[d];
      }
      for (int d = 0; d < dh; ++d) ot[d] /= sum;
      if (lse) lse[(size_t)j * T + t] = mx + log(sum);
    }
  }
  return 0;
}

int win_oracle_bwd(int B, int h, int dh, int w, const int64_t* off, const float* q,
                   const float* k, const float* v, const float* dout, double scale, double* dq,
                   double* dk, double* dv, int nthreads) {
  if (!valid(B, h, dh, w, off) || !q || !k || !v || !dout || !dq || !dk || !dv) return -1;
  const int64_t T = off[B];
  memset(dq, 0, sizeof(double) * (size_t)T * h * dh);
  memset(dk, 0, sizeof(double) * (size_t)T * h * dh);
  memset(dv, 0, sizeof(double) * (size_t)T * h * dh);
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (long u = 0; u < (long)B * h; ++u) {
    const int b = (int)(u / h), j = (int)(u % h);
    double* P = (double*)malloc(sizeof(double) * (size_t)w);
    double* dP = (double*)malloc(sizeof(double) * (size_t)w);
    if (!P || !dP) {
      free(P); free(dP);
      failed |= 1;
      continue;
    }
    for (int64_t t = off[b]; t < off[b + 1]; ++t) {
      const int64_t lo = window_lo(t, off[b], w);
      const int n = (int)(t - lo + 1);
      const float* qt = q + ((size_t)t * h + j) * dh;
      const float* gt = dout + ((size_t)t * h + j) * dh;
      double mx = -INFINITY;
      for (int i = 0; i < n; ++i) {
        P[i] = scale * dot(qt, k + ((size_t)(lo + i) * h + j) * dh, dh);
        mx = P[i] > mx ? P[i] : mx;
      }
      double sum = 0.0;
      for (int i = 0; i < n; ++i) sum += exp(P[i] - mx);
      double D = 0.0;
      for (int i = 0; i < n; ++i) {
        P[i] = exp(P[i] - mx) / sum;
        dP[i] = dot(gt, v + ((size_t)(lo + i) * h + j) * dh, dh);
        D += P[i] * dP[i];
      }
      double* dqt = dq + ((size_t)t * h + j) * dh;
      for (int i = 0; i < n; ++i) {
        const double dA = P[i] * (dP[i] - D);
        const size_t at = ((size_t)(lo + i) * h + j) * dh;
        for (int d = 0; d < dh; ++d) {
          dqt[d] += scale * dA * (double)k[at + d];
          dk[at + d] += scale * dA * (double)qt[d];
          dv[at + d] += P[i] * (double)gt[d];
        }
      }
    }
    free(P); free(dP);
  }
  return failed ? -2 : 0;
}
