/*
 * Weight Generation oracle: plain, slow, fp64 CPU implementation of the step
 * that produces GDPA's per-sample keys and values from the non-sequential
 * context.  TEST INFRASTRUCTURE ONLY: the tests call it; the product library
 * never does, and this file shares no code, header or constant with it.
 *
 * What it computes.  The Kunlun summary (gist.science, "Resumen Tecnico:
 * Kunlun", section 2.1) lists Weight Generation in the Interaction Block, and
 * the RecSysChannel review ("Kunlun ... [2/2]", item 1) says that K and V are
 * obtained from the context features.  Neither page prints the map.  The
 * plainest reading (R20) is a learned linear map per output tensor: for every
 * sample b with context vector c_b (C values),
 *
 *   Y[b, f] = sum_c W[f, c] * c_b[c],      f in [0, F),  F = h * m * dh,
 *
 * so that Y[b] reshaped to [h, m, dh] is K_b (or V_b, with its own W).  Its
 * gradient for an upstream dY:
 *
 *   dW[f, c]  = sum_b dY[b, f] * c_b[c],    dc_b[c] = sum_f dY[b, f] * W[f, c].
 *
 * Every sum is a plain loop accumulated in double; nothing is blocked, fused
 * or reordered.  Layouts: W [F, C], ctx [B, C], Y and dY [B, F], dW [F, C],
 * dctx [B, C], all row-major.
 */
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Forward.  Returns 0, or -1 on bad arguments. */
int wg_oracle_fwd(int B, int64_t F, int C, const float* W, const float* ctx, double* y,
                  int nthreads) {
  if (B < 0 || F < 0 || C <= 0 || !W || !ctx || !y) return -1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
#pragma omp parallel for schedule(static)
  for (int64_t f = 0; f < F; ++f)
    for (int b = 0; b < B; ++b) {
      double acc = 0.0;
      for (int c = 0; c < C; ++c) acc += (double)W[f * C + c] * (double)ctx[(int64_t)b * C + c];
      y[(int64_t)b * F + f] = acc;
    }
  return 0;
}

/* Backward.  dW [F, C] and dctx [B, C]; either may be NULL (not computed). */
int wg_oracle_bwd(int B, int64_t F, int C, const float* W, const float* ctx, const float* dy,
                  double* dW, double* dctx, int nthreads) {
  if (B < 0 || F < 0 || C <= 0 || !W || !ctx || !dy) return -1;
#ifdef _OPENMP
  if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
  if (dW) {
#pragma omp parallel for schedule(static)
    for (int64_t f = 0; f < F; ++f)
      for (int c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int b = 0; b < B; ++b)
          acc += (double)dy[(int64_t)b * F + f] * (double)ctx[(int64_t)b * C + c];
        dW[f * C + c] = acc;
      }
  }
  if (dctx) {
#pragma omp parallel for schedule(static)
    for (int b = 0; b < B; ++b)
      for (int c = 0; c < C; ++c) {
        double acc = 0.0;
        for (int64_t f = 0; f < F; ++f)
          acc += (double)dy[(int64_t)b * F + f] * (double)W[f * C + c];
        dctx[(int64_t)b * C + c] = acc;
      }
  }
  return 0;
}
