/*
 * GDPA oracle: plain, slow, fp64 CPU implementation of Generalized Dot-Product
 * Attention.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * benchmark's CPU-baseline leg call it; the product library never does, and
 * this file shares no code, header or constant with it.
 *
 * What it computes.  The Kunlun summary (gist.science, "Resumen Tecnico:
 * Kunlun", section 2.2, GDPA bullet) recasts the Personalized FFN as a
 * multi-head attention operator whose queries are the sequence tokens and
 * whose keys and values are weights derived from the non-sequential context;
 * the RecSysChannel review ("Kunlun ... [2/2]", items 1 and 2) adds that K and
 * V come from the context features and the event sequence is turned into Q.
 * Neither page prints a formula.  The plainest reading, which this oracle
 * writes out, is, for every sample b and head j, with
 *   Q^ = Q[off[b]:off[b+1], j, :]   (n_b x dh),
 *   K^ = K[b, j], V^ = V[b, j]       (m x dh):
 *
 *   S  = s * Q^ K^T                  (n_b x m)
 *   P  = phi(S)                      phi in {identity, SiLU, row softmax,
 *                                               ReLU, GELU}
 *   O  = P V^                        (n_b x dh)
 *   LSE_i = M_i + ln sum_k exp(S_ik - M_i),  M_i = max_k S_ik  (softmax)
 *
 * and its gradient for an upstream dO:
 *
 *   dV = P^T dO^,  dP = dO^ V^T,
 *   dS = dP                                   (identity)
 *      = dP * sig(S) (1 + S (1 - sig(S)))     (SiLU, sig = logistic)
 *      = P * (dP - D),  D_i = sum_k P_ik dP_ik (softmax)
 *      = dP * [S > 0]                          (ReLU)
 *      = dP * (Phi(S) + S pdf(S))              (GELU = S Phi(S), Phi the standard
 *                                               normal CDF, pdf its density)
 *   dQ^ = s dS K^,  dK^ = s dS^T Q^.
 *
 * Every dot product is a plain loop accumulated in double.  Inputs are float
 * arrays holding the exact values of the (bf16 or fp32) inputs.  Units
 * (b, j) are independent and run under OpenMP; inside a unit nothing is
 * blocked, fused or reordered.
 *
 * Biased variant (the PFFN with biases, phi(s Q K^T + b1) V + b2; the pages
 * leave the PFFN's biases open, this is reading R19): per sample and head a
 * key bias b1^ = b1[b, j] (m) added to every row of the scaled logits before
 * phi, and an output bias b2^ = b2[b, j] (dh) added to every row of O:
 *
 *   S  = s * Q^ K^T + 1 b1^T,   O = phi(S) V^ + 1 b2^T,
 *   db1^ = sum_i dS_i.,  db2^ = sum_i dO^_i.   (the other gradients unchanged
 *                                               in form, with this S)
 *
 * Layouts: q, o, dout, dq: [T, h, dh];  k, v, dk, dv: [B, h, m, dh];
 * b1, db1: [B, h, m];  b2, db2: [B, h, dh];
 * offsets: int64 [B+1];  lse: [h, T].  phi: 0 identity, 1 SiLU, 2 softmax,
 * 3 ReLU, 4 GELU.  ReLU and GELU are the "other phi" of the PFFN variants the
 * Kunlun pages leave open; GELU is taken in its exact form x Phi(x) (reading:
 * the pages name no approximation).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define PHI_IDENTITY 0
#define PHI_SILU 1
#define PHI_SOFTMAX 2
#define PHI_RELU 3
#define PHI_GELU 4

/* Standard normal CDF and density (for GELU): Phi(x) = (1 + erf(x / sqrt 2)) / 2. */
static double normal_cdf(double x) { return 0.5 * (1.0 + erf(x * 0.70710678118654752440)); }
static double normal_pdf(double x) { return 0.39894228040143267794 * exp(-0.5 * x * x); }

static double logistic(double x) { return 1.0 / (1.0 + exp(-x)); }

/* S = s Q^ K^T (+ b1^ on every row when b1b is not NULL) for one unit; S is
 * n x m, row-major. */
static void logits(int n, int m, int dh, int h, const float* qb, const float* kb,
                   const float* b1b, double scale, double* S) {
  for (int i = 0; i < n; ++i) {
    const float* qi = qb + (size_t)i * h * dh;
    for (int k = 0; k < m; ++k) {
      const float* kk = kb + (size_t)k * dh;
      double acc = 0.0;
      for (int d = 0; d < dh; ++d) acc += (double)qi[d] * (double)kk[d];
      S[(size_t)i * m + k] = scale * acc + (b1b ? (double)b1b[k] : 0.0);
    }
  }
}

/* P = phi(S) in place of a separate array; for softmax also the row LSE. */
static void activation(int n, int m, int phi, const double* S, double* P, double* lse_rows) {
  for (int i = 0; i < n; ++i) {
    const double* si = S + (size_t)i * m;
    double* pi = P + (size_t)i * m;
    if (phi == PHI_IDENTITY) {
      for (int k = 0; k < m; ++k) pi[k] = si[k];
    } else if (phi == PHI_SILU) {
      for (int k = 0; k < m; ++k) pi[k] = si[k] / (1.0 + exp(-si[k]));
    } else if (phi == PHI_RELU) {
      for (int k = 0; k < m; ++k) pi[k] = si[k] > 0.0 ? si[k] : 0.0;
    } else if (phi == PHI_GELU) {
      for (int k = 0; k < m; ++k) pi[k] = si[k] * normal_cdf(si[k]);
    } else {
      double mx = -INFINITY;
      for (int k = 0; k < m; ++k) mx = si[k] > mx ? si[k] : mx;
      double sum = 0.0;
      for (int k = 0; k < m; ++k) sum += exp(si[k] - mx);
      for (int k = 0; k < m; ++k) pi[k] = exp(si[k] - mx) / sum;
      if (lse_rows) lse_rows[i] = mx + log(sum);
    }
  }
}

static int valid_args(int B, int h, int dh, int m, const int64_t* offsets) {
  if (B < 0 || h <= 0 || dh <= 0 || m <= 0 || !offsets) return 0;
  if (offsets[0] != 0) return 0;
  for (int b = 0; b < B; ++b)
    if (offsets[b + 1] < offsets[b]) return 0;
  return 1;
}

/* Forward.  o: [T,h,dh] (required), lse: [h,T] (softmax only; may be NULL);
 * b1 [B,h,m] and b2 [B,h,dh] may be NULL (no bias).
 * Returns 0 on success, -1 on bad arguments, -2 if memory ran out. */
int gdpa_oracle_fwd_bias(int B, int h, int dh, int m, const int64_t* offsets,
                         const float* q, const float* k, const float* v, const float* b1,
                         const float* b2, int phi, double scale, double* o, double* lse,
                         int nthreads) {
  if (!valid_args(B, h, dh, m, offsets) || phi < 0 || phi > 4 || !q || !k || !v || !o)
    return -1;
  const int64_t T = offsets[B];
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (long u = 0; u < (long)B * h; ++u) {
    const int b = (int)(u / h), j = (int)(u % h);
    const int64_t t0 = offsets[b];
    const int n = (int)(offsets[b + 1] - t0);
    if (n == 0) continue;
    double* S = (double*)malloc(sizeof(double) * (size_t)n * m);
    double* P = (double*)malloc(sizeof(double) * (size_t)n * m);
    double* L = (double*)malloc(sizeof(double) * (size_t)n);
    if (!S || !P || !L) {
      free(S); free(P); free(L);
      failed |= 1;
      continue;
    }
    const float* qb = q + ((size_t)t0 * h + j) * dh;
    const float* kb = k + ((size_t)b * h + j) * (size_t)m * dh;
    const float* vb = v + ((size_t)b * h + j) * (size_t)m * dh;
    const float* b1b = b1 ? b1 + ((size_t)b * h + j) * (size_t)m : NULL;
    const float* b2b = b2 ? b2 + ((size_t)b * h + j) * (size_t)dh : NULL;
    logits(n, m, dh, h, qb, kb, b1b, scale, S);
    activation(n, m, phi, S, P, L);
    for (int i = 0; i < n; ++i) {
      double* oi = o + ((size_t)(t0 + i) * h + j) * dh;
      for (int d = 0; d < dh; ++d) {
        double acc = 0.0;
        for (int kk = 0; kk < m; ++kk) acc += P[(size_t)i * m + kk] * (double)vb[(size_t)kk * dh + d];
        oi[d] = acc + (b2b ? (double)b2b[d] : 0.0);
      }
      if (lse && phi == PHI_SOFTMAX) lse[(size_t)j * T + t0 + i] = L[i];
    }
    free(S); free(P); free(L);
  }
  return failed ? -2 : 0;
}

/* Backward.  dout: [T,h,dh]; dq: [T,h,dh]; dk, dv: [B,h,m,dh] (all required).
 * b1 [B,h,m] may be NULL (no key bias; b2 does not enter the gradients);
 * db1 [B,h,m] and db2 [B,h,dh] are written when not NULL.
 * P is recomputed from its definition; no forward state is taken. */
int gdpa_oracle_bwd_bias(int B, int h, int dh, int m, const int64_t* offsets,
                         const float* q, const float* k, const float* v, const float* b1,
                         const float* dout, int phi, double scale, double* dq, double* dk,
                         double* dv, double* db1, double* db2, int nthreads) {
  if (!valid_args(B, h, dh, m, offsets) || phi < 0 || phi > 4 || !q || !k || !v ||
      !dout || !dq || !dk || !dv)
    return -1;
  int failed = 0;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(dynamic, 1) reduction(| : failed)
  for (long u = 0; u < (long)B * h; ++u) {
    const int b = (int)(u / h), j = (int)(u % h);
    const int64_t t0 = offsets[b];
    const int n = (int)(offsets[b + 1] - t0);
    const float* qb = q + ((size_t)t0 * h + j) * dh;
    const float* kb = k + ((size_t)b * h + j) * (size_t)m * dh;
    const float* vb = v + ((size_t)b * h + j) * (size_t)m * dh;
    const float* gb = dout + ((size_t)t0 * h + j) * dh;
    double* dkb = dk + ((size_t)b * h + j) * (size_t)m * dh;
    double* dvb = dv + ((size_t)b * h + j) * (size_t)m * dh;
    const float* b1b = b1 ? b1 + ((size_t)b * h + j) * (size_t)m : NULL;
    double* db1b = db1 ? db1 + ((size_t)b * h + j) * (size_t)m : NULL;
    double* db2b = db2 ? db2 + ((size_t)b * h + j) * (size_t)dh : NULL;
    memset(dkb, 0, sizeof(double) * (size_t)m * dh);
    memset(dvb, 0, sizeof(double) * (size_t)m * dh);
    if (db1b) memset(db1b, 0, sizeof(double) * (size_t)m);
    if (db2b) memset(db2b, 0, sizeof(double) * (size_t)dh);
    if (n == 0) continue;
    /* db2^ = sum_i dO^_i. */
    if (db2b)
      for (int d = 0; d < dh; ++d) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += (double)gb[(size_t)i * h * dh + d];
        db2b[d] = acc;
      }
    double* S = (double*)malloc(sizeof(double) * (size_t)n * m);
    double* P = (double*)malloc(sizeof(double) * (size_t)n * m);
    double* dP = (double*)malloc(sizeof(double) * (size_t)n * m);
    if (!S || !P || !dP) {
      free(S); free(P); free(dP);
      failed |= 1;
      continue;
    }
    logits(n, m, dh, h, qb, kb, b1b, scale, S);
    activation(n, m, phi, S, P, NULL);
    /* dP = dO^ V^T */
    for (int i = 0; i < n; ++i)
      for (int kk = 0; kk < m; ++kk) {
        double acc = 0.0;
        for (int d = 0; d < dh; ++d)
          acc += (double)gb[(size_t)i * h * dh + d] * (double)vb[(size_t)kk * dh + d];
        dP[(size_t)i * m + kk] = acc;
      }
    /* dV = P^T dO^ */
    for (int kk = 0; kk < m; ++kk)
      for (int d = 0; d < dh; ++d) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += P[(size_t)i * m + kk] * (double)gb[(size_t)i * h * dh + d];
        dvb[(size_t)kk * dh + d] = acc;
      }
    /* dS, overwriting dP */
    for (int i = 0; i < n; ++i) {
      double* dpi = dP + (size_t)i * m;
      const double* si = S + (size_t)i * m;
      const double* pi = P + (size_t)i * m;
      if (phi == PHI_SILU) {
        for (int kk = 0; kk < m; ++kk) {
          const double sg = logistic(si[kk]);
          dpi[kk] = dpi[kk] * sg * (1.0 + si[kk] * (1.0 - sg));
        }
      } else if (phi == PHI_RELU) {
        for (int kk = 0; kk < m; ++kk) dpi[kk] = si[kk] > 0.0 ? dpi[kk] : 0.0;
      } else if (phi == PHI_GELU) {
        for (int kk = 0; kk < m; ++kk)
          dpi[kk] = dpi[kk] * (normal_cdf(si[kk]) + si[kk] * normal_pdf(si[kk]));
      } else if (phi == PHI_SOFTMAX) {
        double D = 0.0;
        for (int kk = 0; kk < m; ++kk) D += pi[kk] * dpi[kk];
        for (int kk = 0; kk < m; ++kk) dpi[kk] = pi[kk] * (dpi[kk] - D);
      }
    }
    /* db1^ = sum_i dS_i. */
    if (db1b)
      for (int kk = 0; kk < m; ++kk) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += dP[(size_t)i * m + kk];
        db1b[kk] = acc;
      }
    /* dQ^ = s dS K^ */
    for (int i = 0; i < n; ++i) {
      double* dqi = dq + ((size_t)(t0 + i) * h + j) * dh;
      for (int d = 0; d < dh; ++d) {
        double acc = 0.0;
        for (int kk = 0; kk < m; ++kk) acc += dP[(size_t)i * m + kk] * (double)kb[(size_t)kk * dh + d];
        dqi[d] = scale * acc;
      }
    }
    /* dK^ = s dS^T Q^ */
    for (int kk = 0; kk < m; ++kk)
      for (int d = 0; d < dh; ++d) {
        double acc = 0.0;
        for (int i = 0; i < n; ++i) acc += dP[(size_t)i * m + kk] * (double)qb[(size_t)i * h * dh + d];
        dkb[(size_t)kk * dh + d] = scale * acc;
      }
    free(S); free(P); free(dP);
  }
  return failed ? -2 : 0;
}

/* The operator without biases. */
int gdpa_oracle_fwd(int B, int h, int dh, int m, const int64_t* offsets, const float* q,
                    const float* k, const float* v, int phi, double scale, double* o,
                    double* lse, int nthreads) {
  return gdpa_oracle_fwd_bias(B, h, dh, m, offsets, q, k, v, NULL, NULL, phi, scale, o, lse,
                              nthreads);
}

int gdpa_oracle_bwd(int B, int h, int dh, int m, const int64_t* offsets, const float* q,
                    const float* k, const float* v, const float* dout, int phi, double scale,
                    double* dq, double* dk, double* dv, int nthreads) {
  return gdpa_oracle_bwd_bias(B, h, dh, m, offsets, q, k, v, NULL, dout, phi, scale, dq, dk, dv,
                              NULL, NULL, nthreads);
}

int gdpa_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
