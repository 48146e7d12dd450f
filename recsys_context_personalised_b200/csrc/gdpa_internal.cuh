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

// Bias terms of the biased variant phi(s Q K^T + b1) V + b2 (each may be NULL):
// b1 [B, h, m] and b2 [B, h, dh] inputs, db1 and db2 (same shapes) outputs; fp32.
struct Bias {
  const float* b1 = nullptr;
  const float* b2 = nullptr;
  float* db1 = nullptr;
  float* db2 = nullptr;
};


// Builds the jagged tile list (tiles of `bm` rows) and clears the status word.
cudaError_t launch_schedule(const gdpa_problem_t& p, const int32_t* offsets, int bm,
                            WsHeader* ws, Tile* tiles, cudaStream_t st);

// Backward list of (sample, head, 128-key block) items, longest samples first.
cudaError_t launch_schedule_kv(const gdpa_problem_t& p, const int32_t* offsets, WsHeader* ws,
                               Tile* tiles, cudaStream_t st);

// Seed-pooling work list (one item per (sample with tokens, pair of heads),
// longest first; B <= 4096) and the outputs of samples without tokens.
// Backward list of the jagged-key variants: (sample, head, 128-token key block)
// items of the samples with tokens, longest samples first (B <= 4096).
cudaError_t launch_schedule_jkv(const int32_t* offsets, int B, int h, int64_t T, int max_n,
                                WsHeader* ws, Tile* tiles, int64_t cap, cudaStream_t st);
cudaError_t launch_schedule_pool(const int32_t* offsets, int B, int h, int64_t T, int max_n,
                                 WsHeader* ws, Tile* tiles, cudaStream_t st);
cudaError_t launch_pool_empty(const int32_t* offsets, int B, int h, int S, int dh, void* o,
                              float* lse, const WsHeader* ws, cudaStream_t st);

// SIMT kernels (fp32 problems only; fp32 math).
cudaError_t launch_simt_fwd(const gdpa_problem_t& p, const void* q, const void* k,
                            const void* v, const Bias& bs, void* o, float* lse, WsHeader* ws,
                            const Tile* tiles, int64_t tile_cap, cudaStream_t st);
cudaError_t launch_row_dot(const gdpa_problem_t& p, const void* o, const void* dout,
                           float* dsum, cudaStream_t st);
cudaError_t launch_simt_bwd_dq(const gdpa_problem_t& p, const void* q, const void* k,
                               const void* v, const Bias& bs, const float* lse, const float* dsum,
                               const void* dout, void* dq, WsHeader* ws, const Tile* tiles,
                               int64_t tile_cap, cudaStream_t st);
cudaError_t launch_simt_bwd_dkdv(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                                 const void* k, const void* v, const Bias& bs, const float* lse,
                                 const float* dsum, const void* dout, void* dk, void* dv,
                                 WsHeader* ws, cudaStream_t st);

// Backward bias terms: db2 = per-sample token sums of dO, softmax row sums
// D = rowsum(dO * (O - b2)) into `dsum` (when not NULL), db1 zeroed (the
// fused kernels add into it).  Skips its work when the scheduler rejected the
// offsets.
cudaError_t launch_bias_prep(const gdpa_problem_t& p, const int32_t* offsets, const void* o,
                             const void* g, const float* b2, float* dsum, float* db1,
                             float* db2, const WsHeader* ws, cudaStream_t st);

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
// with derivative Phi(x) + x * exp(-x^2/2) / sqrt(2 pi) (erf to 3.4e-6, below).
__device__ __forceinline__ float relu_f(float x) { return fmaxf(x, 0.f); }
__device__ __forceinline__ float relu_grad(float x) { return x > 0.f ? 1.f : 0.f; }
// GELU without the MUFU unit: x Phi(x) = x / 2 + |x| t h(t^2), t = min(|x| / sqrt 2, Z),
// h(u) = erf(sqrt u) / (2 sqrt u), with h a degree-12 polynomial in the centred variable
// s = 2 t^2 / Z^2 - 1 (interpolation at the Chebyshev-Lobatto points, with erf(Z) := 1;
// gelu_fit.py in the package reproduces the coefficients).  Largest error of the fp32
// evaluation against the exact GELU on [-10, 10]: 3.4e-6 (absolute).
constexpr float kGeluZ = 3.6f;
static __constant__ float kGeluH[13] = {0.19635604321956635f, -0.09774208813905716f, 0.07190582156181335f, -0.05697321519255638f, 0.04490869492292404f, -0.0334814228117466f, 0.024110063910484314f, -0.0178938377648592f, 0.0107343140989542f, -0.0034032068215310574f, 0.002155375201255083f, -0.0031565739773213863f, 0.0013689183397218585f};
// t * h(t^2) = erf(t) / 2 for t = min(|x| / sqrt 2, Z)
__device__ __forceinline__ float half_erf_abs(float ax) {
  const float t = fminf(ax * 0.7071067811865476f, kGeluZ);
  const float s = fmaf(t * t, 2.f / (kGeluZ * kGeluZ), -1.f);
  float p = kGeluH[12];
#pragma unroll
  for (int k = 11; k >= 0; --k) p = fmaf(p, s, kGeluH[k]);
  return t * p;
}
__device__ __forceinline__ float gelu_f(float x) {
  return fmaf(fabsf(x), half_erf_abs(fabsf(x)), 0.5f * x);
}
// dGELU/dx = Phi(x) + x exp(-x^2/2) / sqrt(2 pi)
__device__ __forceinline__ float gelu_grad(float x) {
  const float cdf = 0.5f + copysignf(half_erf_abs(fabsf(x)), x);
  return fmaf(x * 0.3989422804014327f, __expf(-0.5f * x * x), cdf);
}
// GELU and its derivative for two values, the polynomial in packed fp32
// arithmetic (the backward's activation)
__device__ __forceinline__ void gelu_fg2(float2 x, float2& p, float2& grad) {
  const float2 ax = make_float2(fabsf(x.x), fabsf(x.y));
  const float2 t = make_float2(fminf(ax.x * 0.7071067811865476f, kGeluZ),
                               fminf(ax.y * 0.7071067811865476f, kGeluZ));
  const float c = 2.f / (kGeluZ * kGeluZ);
  const float2 s = __ffma2_rn(__fmul2_rn(t, t), make_float2(c, c), make_float2(-1.f, -1.f));
  float2 q = make_float2(kGeluH[12], kGeluH[12]);
#pragma unroll
  for (int k = 11; k >= 0; --k) q = __ffma2_rn(q, s, make_float2(kGeluH[k], kGeluH[k]));
  const float2 h = __fmul2_rn(t, q);                       // erf(|x| / sqrt 2) / 2
  p = __ffma2_rn(ax, h, __fmul2_rn(x, make_float2(0.5f, 0.5f)));
  const float2 cdf = make_float2(0.5f + copysignf(h.x, x.x), 0.5f + copysignf(h.y, x.y));
  const float2 gauss = make_float2(__expf(-0.5f * x.x * x.x), __expf(-0.5f * x.y * x.y));
  grad = __ffma2_rn(__fmul2_rn(x, make_float2(0.3989422804014327f, 0.3989422804014327f)), gauss,
                    cdf);
}
// GELU of two values with packed fp32 arithmetic (the forward's activation)
__device__ __forceinline__ float2 gelu_f2(float2 x) {
  const float2 ax = make_float2(fabsf(x.x), fabsf(x.y));
  const float2 t = make_float2(fminf(ax.x * 0.7071067811865476f, kGeluZ),
                               fminf(ax.y * 0.7071067811865476f, kGeluZ));
  const float c = 2.f / (kGeluZ * kGeluZ);
  const float2 s = __ffma2_rn(__fmul2_rn(t, t), make_float2(c, c), make_float2(-1.f, -1.f));
  float2 p = make_float2(kGeluH[12], kGeluH[12]);
#pragma unroll
  for (int k = 11; k >= 0; --k) p = __ffma2_rn(p, s, make_float2(kGeluH[k], kGeluH[k]));
  return __ffma2_rn(__fmul2_rn(ax, t), p, __fmul2_rn(x, make_float2(0.5f, 0.5f)));
}

// 2^x for two values at once on the FMA pipe, without the MUFU unit: Cody-Waite
// range reduction x = n + f with n = floor(x) and f in [0, 1), 2^f from a
// degree-3 polynomial, and 2^n added into the exponent field.  The polynomial
// minimises the largest relative error |p(f) / 2^f - 1| over [0, 1] (Remez
// exchange, exp2_fit.py in the package, which reproduces these coefficients):
// the error is at most 7.5e-5, well below half an ulp of bf16 (2^-9), the
// precision of the P operand it feeds.  x is clamped at -126 so that the
// biased exponent of the result stays >= 0 (every x <= -126 gives about
// 2^-126, negligible next to a row sum >= 1); x must be < 127.
constexpr float kExp2C0 = 0.99992520f, kExp2C1 = 0.69583356f, kExp2C2 = 0.22606716f,
                kExp2C3 = 0.07802452f;
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
  x.x = fmaxf(x.x, -126.f);
  x.y = fmaxf(x.y, -126.f);
  const float2 t = __fadd2_rd(x, make_float2(12582912.f, 12582912.f));   // 1.5 * 2^23 + floor(x)
  const float2 n = __fadd2_rn(t, make_float2(-12582912.f, -12582912.f));  // floor(x), exact
  const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);             // x - floor(x), exact
  float2 q = __ffma2_rn(f, make_float2(kExp2C3, kExp2C3), make_float2(kExp2C2, kExp2C2));
  q = __ffma2_rn(q, f, make_float2(kExp2C1, kExp2C1));
  q = __ffma2_rn(q, f, make_float2(kExp2C0, kExp2C0));
  // the low bits of t hold n (1.5 * 2^23 has an ulp of 1): n << 23 scales q by 2^n
  return make_float2(__uint_as_float(__float_as_uint(q.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(q.y) + (__float_as_uint(t.y) << 23)));
}

}  // namespace gdpa
