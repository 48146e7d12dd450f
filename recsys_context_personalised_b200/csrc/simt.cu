// SIMT (CUDA-core FFMA) GDPA kernels: the exact-fp32 path, the only path of
// fp32 problems (tensor-core formats are too coarse for fp32 parity); bf16
// problems run on the tcgen05 kernels only.
//
// Operator (Kunlun summary, section 2.2, GDPA bullet; RecSysChannel review
// "Kunlun ... [2/2]", items 1-2): per sample b and head j,
//   S = s Q K^T, P = phi(S), O = P V, with phi in {identity, SiLU, softmax,
//   ReLU, GELU};
// backward: dV = P^T dO, dP = dO V^T, dS = dP * phi'(S) (softmax:
// P * (dP - D), D = rowsum(dO * O)), dQ = s dS K, dK = s dS^T Q.
//
// Thread layout of every kernel: 256 threads own a 64-row block; row r =
// tid / 4 is shared by the 4 consecutive lanes c = tid % 4, which each own
// dh/4 output columns and 8 of every 32-wide chunk of the inner index.
#include <math.h>

#include "gdpa_internal.cuh"

namespace gdpa {
namespace {

constexpr int kThreads = 256;
constexpr int kRows = 64;    // rows (query tokens or keys) per block
constexpr int kChunk = 32;   // inner-index chunk (keys or tokens)

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }
__device__ __forceinline__ float silu_grad(float x) {
  const float sg = 1.0f / (1.0f + expf(-x));
  return sg * (1.0f + x * (1.0f - sg));
}

template <typename T, int DH>
__global__ void __launch_bounds__(kThreads)
simt_fwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                const float* __restrict__ b1, const float* __restrict__ b2,
                T* __restrict__ o, float* __restrict__ lse, int64_t Ttot, int h, int m, int phi,
                float scale, const WsHeader* __restrict__ ws, const Tile* __restrict__ tiles) {
  if ((int)blockIdx.x >= ws->tile_count) return;
  const Tile tl = tiles[blockIdx.x];
  extern __shared__ float smem[];
  constexpr int LD = DH + 1, CW = DH / 4, PL = kChunk + 1;
  float* Qs = smem;                 // [kRows][LD]
  float* Ks = Qs + kRows * LD;      // [kChunk][LD]
  float* Vs = Ks + kChunk * LD;     // [kChunk][DH]
  float* Ps = Vs + kChunk * DH;     // [kRows][PL]
  const int tid = threadIdx.x, r = tid >> 2, c = tid & 3;
  for (int i = tid; i < kRows * DH; i += kThreads) {
    const int rr = i / DH, d = i % DH;
    float x = 0.f;
    if (rr < tl.rows) x = Elem<T>::to_f(q[((int64_t)(tl.row0 + rr) * h + tl.head) * DH + d]);
    Qs[rr * LD + d] = x;
  }
  const T* kb = k + ((int64_t)tl.b * h + tl.head) * (int64_t)m * DH;
  const T* vb = v + ((int64_t)tl.b * h + tl.head) * (int64_t)m * DH;
  const float* b1r = b1 ? b1 + ((int64_t)tl.b * h + tl.head) * m : nullptr;
  float acc[CW];
#pragma unroll
  for (int j = 0; j < CW; ++j) acc[j] = 0.f;
  float mrun = -INFINITY, lrun = 0.f;
  for (int k0 = 0; k0 < m; k0 += kChunk) {
    __syncthreads();
    for (int i = tid; i < kChunk * DH; i += kThreads) {
      const int kk = i / DH, d = i % DH;
      float xk = 0.f, xv = 0.f;
      if (k0 + kk < m) {
        xk = Elem<T>::to_f(kb[(int64_t)(k0 + kk) * DH + d]);
        xv = Elem<T>::to_f(vb[(int64_t)(k0 + kk) * DH + d]);
      }
      Ks[kk * LD + d] = xk;
      Vs[kk * DH + d] = xv;
    }
    __syncthreads();
    float s[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float* kr = Ks + (c * 8 + i) * LD;
      const float* qr = Qs + r * LD;
      float dot = 0.f;
#pragma unroll 8
      for (int d = 0; d < DH; ++d) dot = fmaf(qr[d], kr[d], dot);
      const int key = k0 + c * 8 + i;
      s[i] = b1r && key < m ? fmaf(scale, dot, b1r[key]) : scale * dot;
    }
    if (phi == GDPA_PHI_SOFTMAX) {
      float cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (k0 + c * 8 + i < m) cm = fmaxf(cm, s[i]);
        else s[i] = -INFINITY;
      }
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
      const float mnew = fmaxf(mrun, cm);
      const float alpha = expf(mrun - mnew);
      float ps = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        s[i] = expf(s[i] - mnew);
        ps += s[i];
      }
      ps += __shfl_xor_sync(0xffffffffu, ps, 1);
      ps += __shfl_xor_sync(0xffffffffu, ps, 2);
      lrun = lrun * alpha + ps;
      mrun = mnew;
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] *= alpha;
    } else if (phi == GDPA_PHI_SILU) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] = silu_f(s[i]);
    } else if (phi == GDPA_PHI_RELU) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] = relu_f(s[i]);
    } else if (phi == GDPA_PHI_GELU) {
#pragma unroll
      for (int i = 0; i < 8; ++i) s[i] = gelu_f(s[i]);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) Ps[r * PL + c * 8 + i] = s[i];
    __syncwarp();
    for (int kk = 0; kk < kChunk; ++kk) {
      const float p = Ps[r * PL + kk];
      const float* vr = Vs + kk * DH + c * CW;
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] = fmaf(p, vr[j], acc[j]);
    }
  }
  if (r < tl.rows) {
    float inv = 1.f;
    if (phi == GDPA_PHI_SOFTMAX) inv = 1.f / lrun;
    T* orow = o + ((int64_t)(tl.row0 + r) * h + tl.head) * DH + c * CW;
    const float* b2r = b2 ? b2 + ((int64_t)tl.b * h + tl.head) * DH + c * CW : nullptr;
#pragma unroll
    for (int j = 0; j < CW; ++j) orow[j] = Elem<T>::from_f(fmaf(acc[j], inv, b2r ? b2r[j] : 0.f));
    if (phi == GDPA_PHI_SOFTMAX && c == 0 && lse != nullptr)
      lse[(int64_t)tl.head * Ttot + tl.row0 + r] = mrun + logf(lrun);
  }
}

// D[head, t] = sum_d dO[t, head, d] * O[t, head, d]: one warp per row.
template <typename T>
__global__ void row_dot_kernel(const T* __restrict__ o, const T* __restrict__ g,
                               float* __restrict__ dsum, int64_t rows, int h, int dh,
                               int64_t Ttot) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t row = warp; row < rows; row += nwarps) {
    float acc = 0.f;
    for (int d = lane; d < dh; d += 32)
      acc = fmaf(Elem<T>::to_f(o[row * dh + d]), Elem<T>::to_f(g[row * dh + d]), acc);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      const int64_t t = row / h;
      const int j = (int)(row % h);
      dsum[(int64_t)j * Ttot + t] = acc;
    }
  }
}

// dS for one logit given dP and the per-row softmax statistics.
__device__ __forceinline__ float dlogit(int phi, float s, float dp, float lse_r, float d_r,
                                        float* p_out) {
  if (phi == GDPA_PHI_SOFTMAX) {
    const float p = expf(s - lse_r);
    *p_out = p;
    return p * (dp - d_r);
  }
  if (phi == GDPA_PHI_SILU) {
    *p_out = silu_f(s);
    return dp * silu_grad(s);
  }
  if (phi == GDPA_PHI_RELU) {
    *p_out = relu_f(s);
    return dp * relu_grad(s);
  }
  if (phi == GDPA_PHI_GELU) {
    *p_out = gelu_f(s);
    return dp * gelu_grad(s);
  }
  *p_out = s;
  return dp;
}

template <typename T, int DH>
__global__ void __launch_bounds__(kThreads)
simt_bwd_dq_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                   const float* __restrict__ b1, const float* __restrict__ lse,
                   const float* __restrict__ dsum,
                   const T* __restrict__ g, T* __restrict__ dq, int64_t Ttot, int h, int m,
                   int phi, float scale, const WsHeader* __restrict__ ws,
                   const Tile* __restrict__ tiles) {
  if ((int)blockIdx.x >= ws->tile_count) return;
  const Tile tl = tiles[blockIdx.x];
  extern __shared__ float smem[];
  constexpr int LD = DH + 1, CW = DH / 4, PL = kChunk + 1;
  float* Qs = smem;               // [kRows][LD]
  float* Gs = Qs + kRows * LD;    // [kRows][LD]
  float* Ks = Gs + kRows * LD;    // [kChunk][LD]
  float* Vs = Ks + kChunk * LD;   // [kChunk][LD]
  float* Ds = Vs + kChunk * LD;   // [kRows][PL]
  const int tid = threadIdx.x, r = tid >> 2, c = tid & 3;
  for (int i = tid; i < kRows * DH; i += kThreads) {
    const int rr = i / DH, d = i % DH;
    float xq = 0.f, xg = 0.f;
    if (rr < tl.rows) {
      const int64_t at = ((int64_t)(tl.row0 + rr) * h + tl.head) * DH + d;
      xq = Elem<T>::to_f(q[at]);
      xg = Elem<T>::to_f(g[at]);
    }
    Qs[rr * LD + d] = xq;
    Gs[rr * LD + d] = xg;
  }
  float lse_r = 0.f, d_r = 0.f;
  if (phi == GDPA_PHI_SOFTMAX && r < tl.rows) {
    lse_r = lse[(int64_t)tl.head * Ttot + tl.row0 + r];
    d_r = dsum[(int64_t)tl.head * Ttot + tl.row0 + r];
  }
  const T* kb = k + ((int64_t)tl.b * h + tl.head) * (int64_t)m * DH;
  const T* vb = v + ((int64_t)tl.b * h + tl.head) * (int64_t)m * DH;
  const float* b1r = b1 ? b1 + ((int64_t)tl.b * h + tl.head) * m : nullptr;
  float acc[CW];
#pragma unroll
  for (int j = 0; j < CW; ++j) acc[j] = 0.f;
  for (int k0 = 0; k0 < m; k0 += kChunk) {
    __syncthreads();
    for (int i = tid; i < kChunk * DH; i += kThreads) {
      const int kk = i / DH, d = i % DH;
      float xk = 0.f, xv = 0.f;
      if (k0 + kk < m) {
        xk = Elem<T>::to_f(kb[(int64_t)(k0 + kk) * DH + d]);
        xv = Elem<T>::to_f(vb[(int64_t)(k0 + kk) * DH + d]);
      }
      Ks[kk * LD + d] = xk;
      Vs[kk * LD + d] = xv;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int kk = c * 8 + i;
      const float* kr = Ks + kk * LD;
      const float* vr = Vs + kk * LD;
      const float* qr = Qs + r * LD;
      const float* gr = Gs + r * LD;
      float sdot = 0.f, pdot = 0.f;
#pragma unroll 8
      for (int d = 0; d < DH; ++d) {
        sdot = fmaf(qr[d], kr[d], sdot);
        pdot = fmaf(gr[d], vr[d], pdot);
      }
      float p;
      const float x = b1r && k0 + kk < m ? fmaf(scale, sdot, b1r[k0 + kk]) : scale * sdot;
      float ds = dlogit(phi, x, pdot, lse_r, d_r, &p);
      if (k0 + kk >= m || r >= tl.rows) ds = 0.f;
      Ds[r * PL + kk] = ds;
    }
    __syncwarp();
    for (int kk = 0; kk < kChunk; ++kk) {
      const float ds = Ds[r * PL + kk];
      const float* kr = Ks + kk * LD + c * CW;
#pragma unroll
      for (int j = 0; j < CW; ++j) acc[j] = fmaf(ds, kr[j], acc[j]);
    }
  }
  if (r < tl.rows) {
    T* out = dq + ((int64_t)(tl.row0 + r) * h + tl.head) * DH + c * CW;
#pragma unroll
    for (int j = 0; j < CW; ++j) out[j] = Elem<T>::from_f(scale * acc[j]);
  }
}

// One block per (sample, head, 64-key tile); loops over the sample's tokens.
template <typename T, int DH>
__global__ void __launch_bounds__(kThreads)
simt_bwd_dkdv_kernel(const T* __restrict__ q, const int32_t* __restrict__ offsets,
                     const T* __restrict__ k, const T* __restrict__ v,
                     const float* __restrict__ b1, float* __restrict__ db1,
                     const float* __restrict__ lse, const float* __restrict__ dsum,
                     const T* __restrict__ g, T* __restrict__ dk, T* __restrict__ dv,
                     int64_t Ttot, int h, int m, int phi, float scale,
                     const WsHeader* __restrict__ ws) {
  if (ws->status == GDPA_ERR_INVALID_ARG) return;
  const int ktiles = (m + kRows - 1) / kRows;
  const int kt = blockIdx.x % ktiles;
  const int head = (blockIdx.x / ktiles) % h;
  const int b = blockIdx.x / (ktiles * h);
  const int key0 = kt * kRows;
  extern __shared__ float smem[];
  constexpr int LD = DH + 1, CW = DH / 4, PL = kChunk + 1;
  float* Ks = smem;                 // [kRows][LD]
  float* Vs = Ks + kRows * LD;      // [kRows][LD]
  float* Qs = Vs + kRows * LD;      // [kChunk][LD]
  float* Gs = Qs + kChunk * LD;     // [kChunk][LD]
  float* Ps = Gs + kChunk * LD;     // [kRows][PL]
  float* Dss = Ps + kRows * PL;     // [kRows][PL]
  float* Ls = Dss + kRows * PL;     // [kChunk]
  float* Dr = Ls + kChunk;          // [kChunk]
  const int tid = threadIdx.x, r = tid >> 2, c = tid & 3;
  const int64_t kvbase = ((int64_t)b * h + head) * (int64_t)m * DH;
  for (int i = tid; i < kRows * DH; i += kThreads) {
    const int rr = i / DH, d = i % DH;
    float xk = 0.f, xv = 0.f;
    if (key0 + rr < m) {
      xk = Elem<T>::to_f(k[kvbase + (int64_t)(key0 + rr) * DH + d]);
      xv = Elem<T>::to_f(v[kvbase + (int64_t)(key0 + rr) * DH + d]);
    }
    Ks[rr * LD + d] = xk;
    Vs[rr * LD + d] = xv;
  }
  const int t0 = offsets[b];
  const int n = offsets[b + 1] - t0;
  // this thread's key bias (row r of the key tile) and its share of db1
  const float b1k = b1 && key0 + r < m ? b1[((int64_t)b * h + head) * m + key0 + r] : 0.f;
  float db1_acc = 0.f;
  float ak[CW], av[CW];
#pragma unroll
  for (int j = 0; j < CW; ++j) ak[j] = av[j] = 0.f;
  for (int i0 = 0; i0 < n; i0 += kChunk) {
    __syncthreads();
    for (int i = tid; i < kChunk * DH; i += kThreads) {
      const int tt = i / DH, d = i % DH;
      float xq = 0.f, xg = 0.f;
      if (i0 + tt < n) {
        const int64_t at = ((int64_t)(t0 + i0 + tt) * h + head) * DH + d;
        xq = Elem<T>::to_f(q[at]);
        xg = Elem<T>::to_f(g[at]);
      }
      Qs[tt * LD + d] = xq;
      Gs[tt * LD + d] = xg;
    }
    if (tid < kChunk) {
      float l = 0.f, dd = 0.f;
      if (phi == GDPA_PHI_SOFTMAX && i0 + tid < n) {
        l = lse[(int64_t)head * Ttot + t0 + i0 + tid];
        dd = dsum[(int64_t)head * Ttot + t0 + i0 + tid];
      }
      Ls[tid] = l;
      Dr[tid] = dd;
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int tt = c * 8 + i;
      const float* kr = Ks + r * LD;
      const float* vr = Vs + r * LD;
      const float* qr = Qs + tt * LD;
      const float* gr = Gs + tt * LD;
      float sdot = 0.f, pdot = 0.f;
#pragma unroll 8
      for (int d = 0; d < DH; ++d) {
        sdot = fmaf(kr[d], qr[d], sdot);
        pdot = fmaf(vr[d], gr[d], pdot);
      }
      float p;
      float ds = dlogit(phi, fmaf(scale, sdot, b1k), pdot, Ls[tt], Dr[tt], &p);
      if (i0 + tt >= n || key0 + r >= m) {
        ds = 0.f;
        p = 0.f;
      }
      db1_acc += ds;
      Ps[r * PL + tt] = p;
      Dss[r * PL + tt] = ds;
    }
    __syncwarp();
    for (int tt = 0; tt < kChunk; ++tt) {
      const float p = Ps[r * PL + tt], ds = Dss[r * PL + tt];
      const float* gr = Gs + tt * LD + c * CW;
      const float* qr = Qs + tt * LD + c * CW;
#pragma unroll
      for (int j = 0; j < CW; ++j) {
        av[j] = fmaf(p, gr[j], av[j]);
        ak[j] = fmaf(ds, qr[j], ak[j]);
      }
    }
  }
  // the 4 lanes of key r each summed dS over 8 of every 32 tokens
  db1_acc += __shfl_xor_sync(0xffffffffu, db1_acc, 1);
  db1_acc += __shfl_xor_sync(0xffffffffu, db1_acc, 2);
  if (db1 && c == 0 && key0 + r < m) db1[((int64_t)b * h + head) * m + key0 + r] = db1_acc;
  if (key0 + r < m) {
    const int64_t at = kvbase + (int64_t)(key0 + r) * DH + c * CW;
#pragma unroll
    for (int j = 0; j < CW; ++j) {
      dv[at + j] = Elem<T>::from_f(av[j]);
      dk[at + j] = Elem<T>::from_f(scale * ak[j]);
    }
  }
}

template <typename T, int DH>
size_t fwd_smem() { return sizeof(float) * (kRows * (DH + 1) + kChunk * (DH + 1) + kChunk * DH + kRows * (kChunk + 1)); }
template <typename T, int DH>
size_t dq_smem() { return sizeof(float) * (2 * kRows * (DH + 1) + 2 * kChunk * (DH + 1) + kRows * (kChunk + 1)); }
template <typename T, int DH>
size_t dkdv_smem() { return sizeof(float) * (2 * kRows * (DH + 1) + 2 * kChunk * (DH + 1) + 2 * kRows * (kChunk + 1) + 2 * kChunk); }

template <typename T, int DH>
cudaError_t fwd_t(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
                  const Bias& bs, void* o, float* lse, WsHeader* ws, const Tile* tiles,
                  int64_t cap, cudaStream_t st) {
  auto kern = simt_fwd_kernel<T, DH>;
  const size_t sm = fwd_smem<T, DH>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  KernelScope ks_("gdpa_simt_fwd", st);
  kern<<<(unsigned)cap, kThreads, sm, st>>>((const T*)q, (const T*)k, (const T*)v, bs.b1, bs.b2,
                                             (T*)o, lse, p.total_tokens, p.h, p.m, p.phi, p.scale,
                                             ws, tiles);
  return cudaGetLastError();
}

template <typename T, int DH>
cudaError_t dq_t(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
                 const Bias& bs, const float* lse, const float* dsum, const void* g, void* dq,
                 WsHeader* ws, const Tile* tiles, int64_t cap, cudaStream_t st) {
  auto kern = simt_bwd_dq_kernel<T, DH>;
  const size_t sm = dq_smem<T, DH>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  KernelScope ks_("gdpa_simt_bwd_dq", st);
  kern<<<(unsigned)cap, kThreads, sm, st>>>((const T*)q, (const T*)k, (const T*)v, bs.b1, lse,
                                             dsum,
                                             (const T*)g, (T*)dq, p.total_tokens, p.h, p.m, p.phi,
                                             p.scale, ws, tiles);
  return cudaGetLastError();
}

template <typename T, int DH>
cudaError_t dkdv_t(const gdpa_problem_t& p, const void* q, const int32_t* offsets, const void* k,
                   const void* v, const Bias& bs, const float* lse, const float* dsum,
                   const void* g, void* dk, void* dv, WsHeader* ws, cudaStream_t st) {
  auto kern = simt_bwd_dkdv_kernel<T, DH>;
  const size_t sm = dkdv_smem<T, DH>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (int64_t)p.B * p.h * ((p.m + kRows - 1) / kRows);
  KernelScope ks_("gdpa_simt_bwd_dkdv", st);
  kern<<<(unsigned)blocks, kThreads, sm, st>>>((const T*)q, offsets, (const T*)k, (const T*)v,
                                                bs.b1, bs.db1, lse, dsum, (const T*)g, (T*)dk, (T*)dv, p.total_tokens,
                                                p.h, p.m, p.phi, p.scale, ws);
  return cudaGetLastError();
}

#define GDPA_DISPATCH_DH(DHV, FN, ...)                                             \
  switch (DHV) {                                                                   \
    case 32: return FN<32>(__VA_ARGS__);                                           \
    case 64: return FN<64>(__VA_ARGS__);                                           \
    case 128: return FN<128>(__VA_ARGS__);                                         \
    default: return cudaErrorInvalidValue;                                         \
  }

template <int DH> cudaError_t fwd_f32(const gdpa_problem_t& p, const void* q, const void* k, const void* v, const Bias& bs, void* o, float* lse, WsHeader* ws, const Tile* t, int64_t cap, cudaStream_t st) { return fwd_t<float, DH>(p, q, k, v, bs, o, lse, ws, t, cap, st); }
template <int DH> cudaError_t dq_f32(const gdpa_problem_t& p, const void* q, const void* k, const void* v, const Bias& bs, const float* l, const float* ds, const void* g, void* dq, WsHeader* ws, const Tile* t, int64_t cap, cudaStream_t st) { return dq_t<float, DH>(p, q, k, v, bs, l, ds, g, dq, ws, t, cap, st); }
template <int DH> cudaError_t dkdv_f32(const gdpa_problem_t& p, const void* q, const int32_t* off, const void* k, const void* v, const Bias& bs, const float* l, const float* ds, const void* g, void* dk, void* dv, WsHeader* ws, cudaStream_t st) { return dkdv_t<float, DH>(p, q, off, k, v, bs, l, ds, g, dk, dv, ws, st); }

}  // namespace

cudaError_t launch_simt_fwd(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
                            const Bias& bs, void* o, float* lse, WsHeader* ws, const Tile* tiles,
                            int64_t cap, cudaStream_t st) {
  if (cap <= 0) return cudaSuccess;
  if (p.dtype != GDPA_DTYPE_F32) return cudaErrorInvalidValue;
  GDPA_DISPATCH_DH(p.dh, fwd_f32, p, q, k, v, bs, o, lse, ws, tiles, cap, st);
}

cudaError_t launch_row_dot(const gdpa_problem_t& p, const void* o, const void* g, float* dsum,
                           cudaStream_t st) {
  const int64_t rows = p.total_tokens * p.h;
  if (rows == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (rows * 32 + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  if (p.dtype != GDPA_DTYPE_F32) return cudaErrorInvalidValue;
  KernelScope ks_("gdpa_row_dot", st);
  row_dot_kernel<float><<<(unsigned)blocks, threads, 0, st>>>((const float*)o, (const float*)g,
                                                              dsum, rows, p.h, p.dh, p.total_tokens);
  return cudaGetLastError();
}

cudaError_t launch_simt_bwd_dq(const gdpa_problem_t& p, const void* q, const void* k,
                               const void* v, const Bias& bs, const float* lse, const float* dsum,
                               const void* g, void* dq, WsHeader* ws, const Tile* tiles,
                               int64_t cap, cudaStream_t st) {
  if (cap <= 0) return cudaSuccess;
  if (p.dtype != GDPA_DTYPE_F32) return cudaErrorInvalidValue;
  GDPA_DISPATCH_DH(p.dh, dq_f32, p, q, k, v, bs, lse, dsum, g, dq, ws, tiles, cap, st);
}

cudaError_t launch_simt_bwd_dkdv(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                                 const void* k, const void* v, const Bias& bs, const float* lse,
                                 const float* dsum, const void* g, void* dk, void* dv,
                                 WsHeader* ws, cudaStream_t st) {
  if (p.dtype != GDPA_DTYPE_F32) return cudaErrorInvalidValue;
  GDPA_DISPATCH_DH(p.dh, dkdv_f32, p, q, offsets, k, v, bs, lse, dsum, g, dk, dv, ws, st);
}

}  // namespace gdpa
