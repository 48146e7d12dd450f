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
constexpr int kChunk = 64;          // tokens per CTA

__global__ void zero_f32_kernel(float* __restrict__ p, int64_t n) {
  const int64_t nth = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += nth) p[i] = 0.f;
}

__device__ __forceinline__ float4 load4(const float* p) {
  return make_float4(p[0], p[1], p[2], p[3]);
}

// Four consecutive elements of a row as floats.
template <typename T> struct Quad;
template <> struct Quad<float> {
  static __device__ __forceinline__ float4 load(const float* p) {
    return *reinterpret_cast<const float4*>(p);
  }
};
template <> struct Quad<__nv_bfloat16> {
  static __device__ __forceinline__ float4 load(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
  }
};

// CTA c takes tokens [c * kChunk, (c + 1) * kChunk) of the jagged batch, all
// heads: the [tokens, h * DH] block is contiguous.  Thread i owns the
// 4-column groups i, i + 256, ... of a token row (h * DH / 4 groups), so every
// load instruction of the CTA reads whole rows.  For each token it adds dO
// into its running db2 columns (flushed with one atomicAdd per column when the
// token's sample changes and at the end) and, for D, the partial dot of dO
// with O - b2 over its 4 columns, reduced over the DH / 4 lanes of a head.
template <typename T, int DH>
__global__ void __launch_bounds__(kBiasThreads)
bias_prep_kernel(const int32_t* __restrict__ offsets, int B, const T* __restrict__ o,
                 const T* __restrict__ g, const float* __restrict__ b2,
                 float* __restrict__ dsum, float* __restrict__ db2, int h, int64_t Ttot,
                 const WsHeader* __restrict__ ws) {
  constexpr int LPH = DH / 4;                       // lanes per head (8, 16 or 32)
  if (ws->status == GDPA_ERR_INVALID_ARG) return;   // offsets rejected by the scheduler
  const int64_t tbeg = (int64_t)blockIdx.x * kChunk;
  if (tbeg >= Ttot) return;
  const int64_t tend = min(tbeg + kChunk, Ttot);
  const int ngrp = h * DH / 4;                      // 4-column groups per token row
  const int lane = threadIdx.x & 31;
  // sample of the first token: the last b with offsets[b] <= tbeg
  int b0 = 0;
  {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((int64_t)offsets[mid] <= tbeg) lo = mid; else hi = mid - 1;
    }
    b0 = lo;
  }
  for (int gi0 = 0; gi0 < ngrp; gi0 += kBiasThreads) {
    const int gi = gi0 + (int)threadIdx.x;           // the whole warp agrees on gi < ngrp
    const bool act = gi < ngrp;
    const int j = act ? gi / LPH : 0;                // head
    const int col = act ? (gi % LPH) * 4 : 0;        // first column within the head
    int b = b0;
    int64_t bend = offsets[b + 1];
    while (bend <= tbeg && b + 1 < B) bend = offsets[++b + 1];
    float4 bias = make_float4(0.f, 0.f, 0.f, 0.f);
    if (act && b2 && dsum) bias = load4(b2 + ((int64_t)b * h + j) * DH + col);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t t = tbeg; t < tend; ++t) {
      if (t >= bend) {                               // next sample (skipping empty ones)
        if (act && db2) {
          float* d = db2 + ((int64_t)b * h + j) * DH + col;
          atomicAdd(d, acc.x); atomicAdd(d + 1, acc.y); atomicAdd(d + 2, acc.z); atomicAdd(d + 3, acc.w);
        }
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
        while (t >= bend && b + 1 < B) bend = offsets[++b + 1];
        if (act && b2 && dsum) bias = load4(b2 + ((int64_t)b * h + j) * DH + col);
      }
      const int64_t at = (t * h + j) * DH + col;
      float4 gv = make_float4(0.f, 0.f, 0.f, 0.f), ov = gv;
      if (act) {
        gv = Quad<T>::load(g + at);
        if (dsum) ov = Quad<T>::load(o + at);
      }
      acc.x += gv.x; acc.y += gv.y; acc.z += gv.z; acc.w += gv.w;
      if (dsum) {
        float dot = gv.x * (ov.x - bias.x);
        dot = fmaf(gv.y, ov.y - bias.y, dot);
        dot = fmaf(gv.z, ov.z - bias.z, dot);
        dot = fmaf(gv.w, ov.w - bias.w, dot);
#pragma unroll
        for (int off = LPH / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
        if (act && lane % LPH == 0) dsum[(int64_t)j * Ttot + t] = dot;
      }
    }
    if (act && db2) {
      float* d = db2 + ((int64_t)b * h + j) * DH + col;
      atomicAdd(d, acc.x); atomicAdd(d + 1, acc.y); atomicAdd(d + 2, acc.z); atomicAdd(d + 3, acc.w);
    }
  }
}

template <typename T>
cudaError_t launch_t(const gdpa_problem_t& p, const int32_t* offsets, const void* o,
                     const void* g, const float* b2, float* dsum, float* db1, float* db2,
                     const WsHeader* ws, cudaStream_t st) {
  // db1 and db2 start at zero: the fused kernels add their per-key sums of dS
  // into db1, and the chunks of this kernel their column sums of dO into db2
  for (int i = 0; i < 2; ++i) {
    float* z = i ? db2 : db1;
    const int64_t n = (int64_t)p.B * p.h * (i ? p.dh : p.m);
    if (!z || n == 0) continue;
    int64_t blocks = (n + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    KernelScope ks_("gdpa_bias_zero", st);
    zero_f32_kernel<<<(unsigned)blocks, 256, 0, st>>>(z, n);
  }
  if ((!dsum && !db2) || p.total_tokens == 0) return cudaGetLastError();
  KernelScope ks_("gdpa_bias_prep", st);
  auto kern = p.dh == 32 ? bias_prep_kernel<T, 32>
                         : p.dh == 64 ? bias_prep_kernel<T, 64> : bias_prep_kernel<T, 128>;
  const int64_t chunks = (p.total_tokens + kChunk - 1) / kChunk;
  kern<<<(unsigned)chunks, kBiasThreads, 0, st>>>(offsets, p.B, (const T*)o, (const T*)g, b2,
                                                 dsum, db2, p.h, p.total_tokens, ws);
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
