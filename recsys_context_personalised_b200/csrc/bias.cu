// Bias terms of the biased PFFN variant phi(s Q K^T + b1) V + b2 that the
// backward needs besides the fused kernels: the output-bias gradient
//   db2[b, j, :] = sum over the tokens t of sample b of dO[t, j, :],
// the softmax row sums D[j, t] = sum_d dO[t, j, d] * (O[t, j, d] - b2[b, j, d])
// (dO . P V, with O the biased forward output), and a zeroed db1 into which
// the fused kernels add their per-key partial sums of dS.
#include "gdpa_internal.cuh"

namespace gdpa {
namespace {

constexpr int kBiasThreads = 256;   // 8 warps

// One CTA per sample: warp w takes the sample's rows w, w + 8, ... of each
// head, lane l the columns l, l + 32, ... (DH / 32 of them).
template <typename T, int DH>
__global__ void __launch_bounds__(kBiasThreads)
bias_prep_kernel(const int32_t* __restrict__ offsets, const T* __restrict__ o,
                 const T* __restrict__ g, const float* __restrict__ b2,
                 float* __restrict__ dsum, float* __restrict__ db1, float* __restrict__ db2,
                 int h, int m, int64_t Ttot, const WsHeader* __restrict__ ws) {
  constexpr int CPL = DH / 32;                      // columns per lane
  __shared__ float part[kBiasThreads / 32][DH];
  if (ws->status == GDPA_ERR_INVALID_ARG) return;   // offsets rejected by the scheduler
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (db1)
    for (int i = threadIdx.x; i < h * m; i += kBiasThreads) db1[(int64_t)b * h * m + i] = 0.f;
  const int t0 = offsets[b], n = offsets[b + 1] - t0;
  for (int j = 0; j < h; ++j) {
    float bias[CPL], acc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      bias[c] = b2 ? b2[((int64_t)b * h + j) * DH + lane + 32 * c] : 0.f;
      acc[c] = 0.f;
    }
    for (int r = warp; r < n; r += kBiasThreads / 32) {
      const int64_t row = ((int64_t)(t0 + r) * h + j) * DH;
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) {
        const float gv = Elem<T>::to_f(g[row + lane + 32 * c]);
        acc[c] += gv;
        if (dsum) dot = fmaf(gv, Elem<T>::to_f(o[row + lane + 32 * c]) - bias[c], dot);
      }
      if (dsum) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (lane == 0) dsum[(int64_t)j * Ttot + t0 + r] = dot;
      }
    }
    if (db2) {
#pragma unroll
      for (int c = 0; c < CPL; ++c) part[warp][lane + 32 * c] = acc[c];
      __syncthreads();
      for (int d = threadIdx.x; d < DH; d += kBiasThreads) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < kBiasThreads / 32; ++w) s += part[w][d];
        db2[((int64_t)b * h + j) * DH + d] = s;
      }
      __syncthreads();
    }
  }
}

template <typename T>
cudaError_t launch_t(const gdpa_problem_t& p, const int32_t* offsets, const void* o,
                     const void* g, const float* b2, float* dsum, float* db1, float* db2,
                     const WsHeader* ws, cudaStream_t st) {
  auto kern = p.dh == 32 ? bias_prep_kernel<T, 32>
                         : p.dh == 64 ? bias_prep_kernel<T, 64> : bias_prep_kernel<T, 128>;
  KernelScope ks_("gdpa_bias_prep", st);
  kern<<<p.B, kBiasThreads, 0, st>>>(offsets, (const T*)o, (const T*)g, b2, dsum, db1, db2, p.h,
                                     p.m, p.total_tokens, ws);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_bias_prep(const gdpa_problem_t& p, const int32_t* offsets, const void* o,
                             const void* g, const float* b2, float* dsum, float* db1,
                             float* db2, const WsHeader* ws, cudaStream_t st) {
  if (!dsum && !db1 && !db2) return cudaSuccess;
  if (p.dtype == GDPA_DTYPE_F32)
    return launch_t<float>(p, offsets, o, g, b2, dsum, db1, db2, ws, st);
  return launch_t<__nv_bfloat16>(p, offsets, o, g, b2, dsum, db1, db2, ws, st);
}

}  // namespace gdpa
