// Internal declarations shared by the GDPA library's translation units.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gdpa.h"

namespace gdpa {

// One work item of a jagged tile list: `rows` query rows of sample `b`,
// head `head`, starting at global token `row0` (rows <= the list's tile size).
struct __align__(16) Tile {
  int32_t b, head, row0, rows;
};

// Workspace header (first 256 bytes of every workspace).
struct __align__(16) WsHeader {
  int32_t status;      // gdpa_status_t detected on the device (sticky per call)
  int32_t tile_count;  // tiles written by the scheduler
  int32_t pad[62];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr int kSimtBM = 64;    // query rows per SIMT tile
constexpr int kMmaBM = 128;    // query rows per tcgen05 tile (TMEM lanes)

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Upper bound of sum_b ceil(n_b / bm) * h given T and B.
inline int64_t tile_capacity(const gdpa_problem_t& p, int bm) {
  return (int64_t)p.h * (p.total_tokens / bm + p.B);
}

// Device-side error reporting: first error wins.
__device__ __forceinline__ void report(WsHeader* ws, int code) {
  atomicCAS(&ws->status, 0, code);
}

// ---------------------------------------------------------------------------
// element conversions
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float x) { return x; }
  static __device__ __forceinline__ float from_f(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float x) { return __float2bfloat16_rn(x); }
};

// ---------------------------------------------------------------------------
// launchers (each returns cudaSuccess or the launch error)

// Builds the jagged tile list (tiles of `bm` rows) and clears the status word.
cudaError_t launch_schedule(const gdpa_problem_t& p, const int32_t* offsets, int bm,
                            WsHeader* ws, Tile* tiles, cudaStream_t st);

// Backward list of (sample, head, 128-key block) items, longest samples first.
cudaError_t launch_schedule_kv(const gdpa_problem_t& p, const int32_t* offsets, WsHeader* ws,
                               Tile* tiles, cudaStream_t st);

// SIMT kernels (fp32 problems only; fp32 math).
cudaError_t launch_simt_fwd(const gdpa_problem_t& p, const void* q, const void* k,
                            const void* v, void* o, float* lse, WsHeader* ws,
                            const Tile* tiles, int64_t tile_cap, cudaStream_t st);
cudaError_t launch_row_dot(const gdpa_problem_t& p, const void* o, const void* dout,
                           float* dsum, cudaStream_t st);
cudaError_t launch_simt_bwd_dq(const gdpa_problem_t& p, const void* q, const void* k,
                               const void* v, const float* lse, const float* dsum,
                               const void* dout, void* dq, WsHeader* ws, const Tile* tiles,
                               int64_t tile_cap, cudaStream_t st);
cudaError_t launch_simt_bwd_dkdv(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                                 const void* k, const void* v, const float* lse,
                                 const float* dsum, const void* dout, void* dk, void* dv,
                                 WsHeader* ws, cudaStream_t st);

// Brackets one kernel launch: counts it for gdpa_last_launch_count() and, while
// gdpa_timing_enable(1) is in force, records CUDA events around it on `st`.
struct KernelScope {
  KernelScope(const char* name, cudaStream_t st);
  ~KernelScope();
  int rec;
  cudaStream_t st;
};

// Elementwise phi of the PFFN variants on a scaled logit x, and dphi/dx:
// ReLU max(x, 0); GELU in its exact form x * Phi(x), Phi(x) = (1 + erf(x/sqrt 2))/2,
// with derivative Phi(x) + x * exp(-x^2/2) / sqrt(2 pi).
__device__ __forceinline__ float relu_f(float x) { return fmaxf(x, 0.f); }
__device__ __forceinline__ float relu_grad(float x) { return x > 0.f ? 1.f : 0.f; }
// Phi(x) and exp(-x^2/2), with erf from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (|error| <= 1.5e-7): for z >= 0,
// erf(z) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-z^2), t = 1 / (1 + p z).
__device__ __forceinline__ void normal_cdf_gauss(float x, float& cdf, float& gauss) {
  const float z = fabsf(x) * 0.7071067811865476f;
  const float t = __fdividef(1.f, fmaf(0.3275911f, z, 1.f));
  const float poly =
      t * fmaf(t, fmaf(t, fmaf(t, fmaf(t, 1.061405429f, -1.453152027f), 1.421413741f),
                       -0.284496736f),
               0.254829592f);
  gauss = __expf(-z * z);
  cdf = 0.5f + copysignf(0.5f * (1.f - poly * gauss), x);
}
__device__ __forceinline__ float gelu_f(float x) {
  float cdf, gauss;
  normal_cdf_gauss(x, cdf, gauss);
  return x * cdf;
}
__device__ __forceinline__ float gelu_grad(float x) {
  float cdf, gauss;
  normal_cdf_gauss(x, cdf, gauss);
  return fmaf(x * 0.3989422804014327f, gauss, cdf);
}

}  // namespace gdpa
