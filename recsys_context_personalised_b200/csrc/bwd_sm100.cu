// Fused GDPA backward for sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// Gradient of O = phi(s Q K^T) V (Kunlun summary, section 2.2, GDPA bullet;
// RecSysChannel review "Kunlun ... [2/2]", items 1-2) for an upstream dO:
//   dV = P^T dO,  dP = dO V^T,  dS = dP * phi'(S)  (softmax: P * (dP - D),
//   D = rowsum(dO * O)),  dQ = s dS K,  dK = s dS^T Q.
// K and V are generated per sample from its context, so dK and dV reduce over
// the tokens of one sample only.
//
// Work item = (sample b, head j, 128-key block); the CTA that owns it loops
// over the sample's 128-row query tiles and keeps dV and dK of its keys in
// TMEM for the whole loop (no atomics for dK/dV).  The products are taken
// transposed, keys on the MMA's M side (TMEM lanes):
//   S^T  = K Q_i^T          A = K (smem, K-major),  B = Q_i (smem, K-major)
//   dP^T = V dO_i^T         A = V,                  B = dO_i
//   P^T, dS^T               activation warps (lane = key), rows >= n_b zeroed
//   dV  += P^T dO_i         A = P^T (TMEM, bf16),   B = dO_i (smem, MN-major)
//   dK  += dS^T Q_i         A = dS^T (smem, K-major), B = Q_i (MN-major)
//   dQ_i = dS K             A = dS (the same smem bytes read MN-major), B = K (MN-major)
// dQ_i (lane = query row) is added into an fp32 workspace; a last kernel
// scales it by s and rounds it to bf16.
//
// One persistent CTA per SM, static round-robin over a work list sorted by
// sample length (longest first).  Two kernels:
//   - dh = 128 (gdpa_bwd_sm100_kernel, 12 warps): warp 0 TMA producer, warp 1
//     MMA issuer, warp 2 TMEM allocator, warps 4-7 and 8-11 the activation
//     groups (halves of each tile's 128 rows), which also drain dQ_i with
//     vector reductions and store dV (group 0) and dK (group 1);
//   - dh <= 64 (gdpa_bwd_half_kernel, 16 warps): a half-tile pipeline with a
//     separate drain warpgroup and bulk tensor copies (described below).
#include <cudaTypedefs.h>
#include <math.h>

#include <type_traits>

#include "gdpa_internal.cuh"
#include "sm100.cuh"

namespace gdpa {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
int device_sm_count();

namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// SiLU and its gradient on a pair of columns, in packed arithmetic: with
// hx = u/2, phi(u) = hx (1 + tanh hx) and dS = dP * sg * (1 + u (1 - sg)),
// sg = logistic(u) = (1 + tanh hx) / 2.
__device__ __forceinline__ void silu_fg2(float2 hx, float2 g, float2& p, float2& ds) {
  const float2 th = make_float2(tanh_approx(hx.x), tanh_approx(hx.y));
  const float2 sg = __ffma2_rn(make_float2(0.5f, 0.5f), th, make_float2(0.5f, 0.5f));
  p = __ffma2_rn(hx, th, hx);
  const float2 t = __ffma2_rn(__fadd2_rn(hx, hx), __fadd2_rn(make_float2(1.f, 1.f),
                                                             make_float2(-sg.x, -sg.y)),
                              make_float2(1.f, 1.f));
  ds = __fmul2_rn(__fmul2_rn(g, sg), t);
}

// ---------------------------------------------------------------- prep / convert

// Zeroes the fp32 dQ workspace (n4 float4s) and, for softmax, writes the row
// sums D = sum_d dO[row, d] * O[row, d] of the `rows` rows of DH elements:
// at D[head, t] for token rows (t, head), or at D[row] when `flat` (the
// pooled outputs [B, h, S, DH]).
template <int DH>
__global__ void bwd_prep_kernel(const uint4* __restrict__ o, const uint4* __restrict__ g,
                                float* __restrict__ dsum, float4* __restrict__ dq_acc,
                                int64_t n4, int64_t rows, int h, int64_t T, int softmax,
                                int flat) {
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nth = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = tid; i < n4; i += nth) dq_acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!softmax) return;
  // D of a (token, head) row: CPR lanes take one 16-byte piece of O and dO
  // each; a warp covers RPW rows per step and U steps per iteration, so that
  // 2U 16-byte loads per thread are in flight.
  constexpr int CPR = DH / 8, RPW = 32 / CPR, U = 4;
  const int lane = threadIdx.x & 31, sub = lane / CPR, piece = lane % CPR;
  const int64_t warp = tid >> 5, nwarps = nth >> 5;
  for (int64_t r0 = warp * (RPW * U); r0 < rows; r0 += nwarps * (RPW * U)) {
    uint4 x[U], y[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int64_t row = r0 + u * RPW + sub;
      x[u] = y[u] = make_uint4(0u, 0u, 0u, 0u);
      if (row < rows) {
        x[u] = o[row * CPR + piece];
        y[u] = g[row * CPR + piece];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t xa[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
      const uint32_t ya[4] = {y[u].x, y[u].y, y[u].z, y[u].w};
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&xa[e]));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ya[e]));
        acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
      }
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const int64_t row = r0 + u * RPW + sub;
      if (piece == 0 && row < rows) dsum[flat ? row : (int64_t)(row % h) * T + row / h] = acc;
    }
  }
}

// x *= s over n floats (the pooled seeds' gradient, accumulated unscaled).
__global__ void scale_f32_kernel(float* __restrict__ x, int64_t n, float scale) {
  const int64_t nth = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += nth) x[i] *= scale;
}

// dQ = bf16(s * dq_acc), 8 elements per thread and iteration.
__global__ void dq_convert_kernel(const float4* __restrict__ acc, uint4* __restrict__ dq,
                                  int64_t n8, float scale) {
  const int64_t nth = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += nth) {
    const float4 a = acc[2 * i], b = acc[2 * i + 1];
    dq[i] = make_uint4(pack_bf16x2(a.x * scale, a.y * scale), pack_bf16x2(a.z * scale, a.w * scale),
                       pack_bf16x2(b.x * scale, b.y * scale), pack_bf16x2(b.z * scale, b.w * scale));
  }
}

// ---------------------------------------------------------------- main kernel

struct BwdArgs {
  const Tile* tiles;
  WsHeader* ws;
  const int32_t* offsets;
  const float* lse;      // [h, T] natural log (softmax)
  const float* dsum;     // [h, T] (softmax)
  float* dq_acc;         // [T, h, dh] fp32
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
  const float* b1;       // [B, h, m] key bias (biased variant; may be NULL)
  float* db1;            // [B, h, m] its gradient, zeroed beforehand (may be NULL)
  int64_t T;
  int h, m;
  int S;                 // seed pooling: seeds per head (query rows of every item)
  int window;            // sliding window: keys t - window < t' <= t
  float scale, scale_log2;
};

// This thread's key bias for the biased variant (zero past m or without b1).
__device__ __forceinline__ float key_bias(const BwdArgs& a, const Tile& it, int key) {
  return a.b1 != nullptr && key < a.m ? __ldg(a.b1 + ((int64_t)it.b * a.h + it.head) * a.m + key)
                                      : 0.f;
}
// Adds this thread's partial sum of dS over its tokens into db1[b, head, key].
__device__ __forceinline__ void add_key_bias_grad(const BwdArgs& a, const Tile& it, int key,
                                                  float acc) {
  if (a.db1 != nullptr && key < a.m)
    atomicAdd(a.db1 + ((int64_t)it.b * a.h + it.head) * a.m + key, acc);
}

template <int DH>
struct BwdCfg {
  static constexpr int CH = DH < 64 ? DH : 64;
  static constexpr int NCH = DH / CH;
  static constexpr uint32_t ROWB = CH * 2;
  static constexpr uint32_t CHUNKB = 128 * ROWB;
  static constexpr uint32_t TILEB = NCH * CHUNKB;          // one [128 x DH] bf16 tile
  static constexpr uint32_t SW = DH < 64 ? kSw64 : kSw128;
  static constexpr uint32_t ATOM = 8 * ROWB;
  static constexpr int NSTG = DH == 128 ? 1 : 2;           // (Q_i, dO_i) stages
  static constexpr uint32_t DSB = 2 * 128 * 128;           // dS^T [128 keys][128 rows] bf16, SW128
  // TMEM columns
  static constexpr uint32_t COL_S = 0, COL_DP = 128, COL_DV = 256, COL_DK = 256 + DH;
  // dh <= 64: two dQ buffers of their own (the drain of step i-1 overlaps the
  // MMAs of step i); dh = 128: one dQ buffer in the dP^T columns.
  static constexpr bool DQ2 = DH <= 64;
  static constexpr uint32_t COL_DQ = DQ2 ? 256 + 2 * DH : COL_DP;
  // barriers
  static constexpr int B_KVFULL = 0, B_KVEMPTY = 1, B_SFULL = 2, B_PFULL = 3, B_DQFULL = 4,
                       B_DQEMPTY = 6, B_ACCFULL = 8, B_ACCEMPTY = 9, B_DRAIN = 10,
                       B_STFULL = 11, B_STEMPTY = 11 + NSTG, NBAR = 11 + 2 * NSTG;
  static constexpr uint32_t OFF_K = 0, OFF_V = TILEB, OFF_STG = 2 * TILEB;
  static constexpr uint32_t OFF_DS = OFF_STG + NSTG * 2 * TILEB;
  // dV/dK epilogue: per activation warp, 32 rows x 64 columns of bf16 (128 B
  // rows), to turn its key rows into whole-row global stores
  static constexpr uint32_t KSTG_WARP = 32 * 128;
  static constexpr uint32_t OFF_KSTG = OFF_DS + DSB;
  static constexpr uint32_t OFF_CTL = OFF_KSTG + 8 * KSTG_WARP;
  static constexpr uint32_t CTL_BYTES = 1024 + 8 * 2 * 128 * 4;  // barriers + per-warp row stats
  static constexpr uint32_t SMEM_USED = 1024 + OFF_CTL + CTL_BYTES;
  static constexpr uint32_t SMEM = SMEM_USED > 120u * 1024u ? SMEM_USED : 120u * 1024u;
  static_assert(SMEM <= 232448u, "exceeds the 227 KB of shared memory a CTA can have");
};

template <int DH, int PHI, bool BIAS>
__global__ void __launch_bounds__(kThreads, 1)
gdpa_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmG,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmDQ, const BwdArgs a) {
  static_assert(DH == 128, "dh <= 64 runs gdpa_bwd_half_kernel");
  using C = BwdCfg<DH>;
  constexpr bool SOFTMAX = PHI == GDPA_PHI_SOFTMAX;
  constexpr uint32_t IDESC_T = idesc_bf16(128, 128, 0, 0);   // S^T, dP^T
  constexpr uint32_t IDESC_KV = idesc_bf16(128, DH, 0, 1);   // dV, dK (B MN-major)
  constexpr uint32_t IDESC_Q = idesc_bf16(128, DH, 1, 1);    // dQ (A and B MN-major)

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sK = base + C::OFF_K, sV = base + C::OFF_V, sStg = base + C::OFF_STG;
  const uint32_t sDS = base + C::OFF_DS;
  uint8_t* ctl = gbase + C::OFF_CTL;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * C::NBAR + 4);
  float* stats = reinterpret_cast<float*>(ctl + 1024);   // [8 warps][2][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(bar(C::B_KVFULL), 1);
    mbar_init(bar(C::B_KVEMPTY), 1);
    mbar_init(bar(C::B_SFULL), 1);
    mbar_init(bar(C::B_PFULL), 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_DQFULL + i), 1);
      mbar_init(bar(C::B_DQEMPTY + i), 256);
    }
    mbar_init(bar(C::B_ACCFULL), 1);
    mbar_init(bar(C::B_ACCEMPTY), 256);
    mbar_init(bar(C::B_DRAIN), 1);
    for (int i = 0; i < C::NSTG; ++i) {
      mbar_init(bar(C::B_STFULL + i), 1);
      mbar_init(bar(C::B_STEMPTY + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmG);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int count = a.ws->status == GDPA_ERR_INVALID_ARG ? 0 : a.ws->tile_count;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t ic = 0, stage = 0, sphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < count; t += gridDim.x) {
        const Tile it = a.tiles[t];
        if (it.rows == 0) continue;
        const int nq = (it.rows + 127) >> 7;
        const int t0 = a.offsets[it.b];
        if (!mbar_wait(bar(C::B_KVEMPTY), (ic & 1u) ^ 1u, abort_flag, kTimeoutNs)) break;
        mbar_expect_tx(bar(C::B_KVFULL), 2 * C::TILEB);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          tma_load_4d(sK + c * C::CHUNKB, &tmK, bar(C::B_KVFULL), c * C::CH, it.row0, it.head, it.b);
          tma_load_4d(sV + c * C::CHUNKB, &tmV, bar(C::B_KVFULL), c * C::CH, it.row0, it.head, it.b);
        }
        for (int i = 0; i < nq; ++i) {
          if (!mbar_wait(bar(C::B_STEMPTY + stage), sphase ^ 1u, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          const uint32_t dst = sStg + stage * 2 * C::TILEB;
          mbar_expect_tx(bar(C::B_STFULL + stage), 2 * C::TILEB);
#pragma unroll
          for (int c = 0; c < C::NCH; ++c) {
            tma_load_3d(dst + c * C::CHUNKB, &tmQ, bar(C::B_STFULL + stage), c * C::CH, it.head,
                        t0 + 128 * i);
            tma_load_3d(dst + C::TILEB + c * C::CHUNKB, &tmG, bar(C::B_STFULL + stage),
                        c * C::CH, it.head, t0 + 128 * i);
          }
          if (++stage == (uint32_t)C::NSTG) {
            stage = 0;
            sphase ^= 1u;
          }
        }
        ++ic;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t ic = 0, stage = 0, sphase = 0, qs = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < count; t += gridDim.x) {
        const Tile it = a.tiles[t];
        if (it.rows == 0) continue;
        const int nq = (it.rows + 127) >> 7;
        if (!mbar_wait(bar(C::B_KVFULL), ic & 1u, abort_flag, kTimeoutNs)) break;
        tc_fence_after();
        for (int i = 0; i < nq; ++i, ++qs) {
          if (!mbar_wait(bar(C::B_STFULL + stage), sphase, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qaddr = sStg + stage * 2 * C::TILEB, gaddr = qaddr + C::TILEB;
          // descriptors built once per group: between two MMAs (whose issue waits
          // for the tensor core) only a constant add remains
          const uint64_t dk0 = smem_desc(sK, 16, C::ATOM, C::SW), dv0 = smem_desc(sV, 16, C::ATOM, C::SW);
          const uint64_t dq0 = smem_desc(qaddr, 16, C::ATOM, C::SW), dg0 = smem_desc(gaddr, 16, C::ATOM, C::SW);
          // S^T = K Q_i^T
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint32_t off = (k / (C::CH / 16)) * C::CHUNKB + (k % (C::CH / 16)) * 32;
            mma_ss(tmem + C::COL_S, desc_advance(dk0, off), desc_advance(dq0, off), IDESC_T,
                   k > 0 ? 1u : 0u);
          }
          // dP^T = V dO_i^T; with one dQ buffer in these columns, dQ_{i-1} must be drained
          if (!C::DQ2 && qs >= 1 &&
              !mbar_wait(bar(C::B_DQEMPTY), (qs - 1) & 1u, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint32_t off = (k / (C::CH / 16)) * C::CHUNKB + (k % (C::CH / 16)) * 32;
            mma_ss(tmem + C::COL_DP, desc_advance(dv0, off), desc_advance(dg0, off), IDESC_T,
                   k > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::B_SFULL));
          if (!mbar_wait(bar(C::B_PFULL), qs & 1u, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          if (i == 0 && !mbar_wait(bar(C::B_ACCEMPTY), (ic & 1u) ^ 1u, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t acc0 = i == 0 ? 0u : 1u;
          const uint64_t gmn0 = smem_desc(gaddr, C::CHUNKB, C::ATOM, C::SW);   // dO_i, MN-major
          const uint64_t qmn0 = smem_desc(qaddr, C::CHUNKB, C::ATOM, C::SW);   // Q_i, MN-major
          const uint64_t dsk0 = smem_desc(sDS, 16, 1024, kSw128);              // dS^T, K-major
          // dV += P^T dO_i   (P^T rows 0-63 in columns 0-31, rows 64-127 in 64-95)
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint32_t acol = C::COL_S + (k < 4 ? 8 * k : 64 + 8 * (k - 4));
            mma_ts(tmem + C::COL_DV, tmem + acol, desc_advance(gmn0, k * 2 * C::ATOM), IDESC_KV,
                   k > 0 ? 1u : acc0);
          }
          // dK += dS^T Q_i
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tmem + C::COL_DK, desc_advance(dsk0, (k >> 2) * 16384 + (k & 3) * 32),
                   desc_advance(qmn0, k * 2 * C::ATOM), IDESC_KV, k > 0 ? 1u : acc0);
          // dQ_i = dS K (into buffer qs % 2 when double-buffered, after its last drain)
          const uint32_t dqb = C::DQ2 ? (qs & 1u) : 0u;
          if (C::DQ2 && !mbar_wait(bar(C::B_DQEMPTY + dqb), ((qs >> 1) & 1u) ^ 1u, abort_flag,
                                   kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t dsm0 = smem_desc(sDS, 16384, 1024, kSw128);           // dS, MN-major
          const uint64_t kmn0 = smem_desc(sK, C::CHUNKB, C::ATOM, C::SW);      // K, MN-major
#pragma unroll
          for (int k = 0; k < 8; ++k)
            mma_ss(tmem + C::COL_DQ + dqb * DH, desc_advance(dsm0, k * 2048),
                   desc_advance(kmn0, k * 2 * C::ATOM), IDESC_Q, k > 0 ? 1u : 0u);
          mma_commit(bar(C::B_STEMPTY + stage));
          mma_commit(bar(C::B_DQFULL + dqb));
          if (++stage == (uint32_t)C::NSTG) {
            stage = 0;
            sphase ^= 1u;
          }
        }
        if (!ok) break;
        mma_commit(bar(C::B_KVEMPTY));
        mma_commit(bar(C::B_ACCFULL));
        ++ic;
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ activation groups
    const int grp = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int lrow = quad * 32 + lane;                 // TMEM lane: key (S^T, dV, dK) or row (dQ)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    float* wst = stats + (warp - 4) * 256;             // this warp's row statistics
    const float c2 = a.scale_log2, sc = a.scale, half_sc = 0.5f * a.scale;
    uint32_t ic = 0, qs = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < count; t += gridDim.x) {
      const Tile it = a.tiles[t];
      const int n = it.rows;
      const int key = it.row0 + lrow;
      __nv_bfloat16* kvout = (grp == 0 ? a.dv : a.dk) +
                             (((int64_t)it.b * a.h + it.head) * a.m + key) * DH;
      if (n == 0) {                                    // no tokens: dK = dV = 0
        if (key < a.m) {
          uint4* d4 = reinterpret_cast<uint4*>(kvout);
#pragma unroll
          for (int c = 0; c < DH / 8; ++c) d4[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      const int nq = (n + 127) >> 7;
      const int t0 = a.offsets[it.b];
      // biased variant: this key's bias (log2 units for softmax, halved for
      // SiLU) and this thread's sum of dS over its tokens (for db1)
      const float b1k = BIAS ? key_bias(a, it, key) : 0.f;
      const float b1l = b1k * 1.4426950408889634f, hb = 0.5f * b1k;
      float db1_acc = 0.f;
      // dQ_i drain: lane = query row of tile i; this group adds half of the columns
      auto drain_dq = [&](int ii, uint32_t step) -> bool {
        const uint32_t b = C::DQ2 ? (step & 1u) : 0u;
        const uint32_t par = C::DQ2 ? ((step >> 1) & 1u) : (step & 1u);
        const bool w = mbar_wait(bar(C::B_DQFULL + b), par, abort_flag, kTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) return false;
        tc_fence_after();
        // Lane = query row.  This group's DH/2 columns go through the warp's
        // shared-memory area, 32 fp32 columns (128 B of a row) at a time, as a
        // swizzled [32 x 32] box that one lane adds into the fp32 accumulator
        // with a bulk tensor reduce-add.  Rows past the sample are exact zeros
        // (their dS is zero): a warp whose rows all lie there adds nothing, and
        // rows past T are clipped by the map.
        const uint32_t kstg = base + C::OFF_KSTG + (uint32_t)(warp - 4) * C::KSTG_WARP;
        const bool adds = 128 * ii + quad * 32 < n;
#pragma unroll
        for (int c0 = 0; c0 < DH / 2; c0 += 32) {
          if (lane == 0) bulk_wait_group_read0();      // the area's last bulk copy has read it
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 32; c += 16) {
            uint32_t v[16];
            tmem_ld_x16(tmem + lane_off + C::COL_DQ + b * DH + grp * (DH / 2) + c0 + c, v);
            tmem_wait_ld();
            if (c0 + c + 16 == DH / 2) {
              tc_fence_before();
              mbar_arrive(bar(C::B_DQEMPTY + b));       // the dQ columns are free
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint32_t chunk = (uint32_t)(c / 4 + j);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                           ::"r"(kstg + lane * 128 + ((chunk ^ (uint32_t)(lane & 7)) << 4)),
                           "r"(v[4 * j]), "r"(v[4 * j + 1]), "r"(v[4 * j + 2]), "r"(v[4 * j + 3])
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (adds && lane == 0) {
            tma_reduce_add_3d(&tmDQ, kstg, grp * (DH / 2) + c0, it.head, t0 + 128 * ii + quad * 32);
            bulk_commit_group();
          }
        }
        return true;
      };
      // softmax row statistics of a query tile, loaded one step ahead
      float nl[2] = {0.f, 0.f}, nd[2] = {0.f, 0.f};
      auto load_stats = [&](int ii) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int rg = 128 * ii + 64 * grp + 32 * u + lane;
          nl[u] = INFINITY;                            // rows past the sample: P = 0
          nd[u] = 0.f;
          if (rg < n) {
            const int64_t at = (int64_t)it.head * a.T + t0 + rg;
            nl[u] = __ldg(a.lse + at);                 // raw: consumed a tile later
            nd[u] = __ldg(a.dsum + at);
          }
        }
      };
      if constexpr (SOFTMAX) load_stats(0);
      for (int i = 0; i < nq; ++i, ++qs) {
        const int rbase = 128 * i + 64 * grp;          // first sample row of this group's half
        if constexpr (SOFTMAX) {
          __syncwarp();
#pragma unroll
          for (int u = 0; u < 2; ++u) {      // -LSE (log2 units) and -D of the 64 rows
            wst[32 * u + lane] = -nl[u] * 1.4426950408889634f;
            wst[64 + 32 * u + lane] = -nd[u];
          }
          __syncwarp();
          if (i + 1 < nq) load_stats(i + 1);
        }
        bool w = mbar_wait(bar(C::B_SFULL), qs & 1u, abort_flag, kTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // FULL: every query row of the group's half lies in the sample, so the
        // activations other than softmax need no row mask either
        auto half_body = [&](auto full_tag) {
          constexpr bool FULL = decltype(full_tag)::value;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            const uint32_t col = 64 * grp + 32 * ch;
            uint32_t s[32], dp[32];
            tmem_ld_x32(tmem + lane_off + C::COL_S + col, s);
            tmem_ld_x32(tmem + lane_off + C::COL_DP + col, dp);
            tmem_wait_ld();
            uint32_t pp[16], dd[16];
            [[maybe_unused]] float4 nl4, nd4;   // softmax: -LSE and -D of rows c..c+3
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              float pv[2], dv2[2];
              [[maybe_unused]] float2 gp, gd;   // phi and dS (GELU: phi') of the pair
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int r = 32 * ch + c + e;
                const float x = __uint_as_float(s[c + e]);
                const float g = __uint_as_float(dp[c + e]);
                float p, ds;
                // u = s x + b1 (the biased logit; b1k = 0 without a key bias)
                if constexpr (SOFTMAX) {
                  if (e == 0) {         // both columns of the pair, in packed arithmetic
                    if ((c & 2) == 0) {   // rows r..r+3 (16-byte aligned)
                      nl4 = *reinterpret_cast<const float4*>(wst + r);
                      nd4 = *reinterpret_cast<const float4*>(wst + 64 + r);
                    }
                    const float2 nlv = (c & 2) ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
                    const float2 ndv = (c & 2) ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
                    const float2 u = __ffma2_rn(
                        make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                        make_float2(c2, c2), BIAS ? __fadd2_rn(nlv, make_float2(b1l, b1l)) : nlv);
                    gp = make_float2(ex2_approx(u.x), ex2_approx(u.y));
                    gd = __fmul2_rn(gp, __fadd2_rn(make_float2(__uint_as_float(dp[c]),
                                                               __uint_as_float(dp[c + 1])),
                                                   ndv));
                  }
                  p = e ? gp.y : gp.x;
                  ds = e ? gd.y : gd.x;
                } else if constexpr (PHI == GDPA_PHI_SILU) {
                  if (e == 0)           // both columns of the pair, in packed arithmetic
                    silu_fg2(__ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                        make_float2(half_sc, half_sc), make_float2(hb, hb)),
                             make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), gp, gd);
                  p = e ? gp.y : gp.x;
                  ds = e ? gd.y : gd.x;
                } else if constexpr (PHI == GDPA_PHI_RELU) {
                  if (e == 0) {         // both columns of the pair, in packed arithmetic
                    const float2 u = __ffma2_rn(
                        make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                        make_float2(sc, sc), make_float2(b1k, b1k));
                    gp = make_float2(relu_f(u.x), relu_f(u.y));
                    gd = __fmul2_rn(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                                    make_float2(relu_grad(u.x), relu_grad(u.y)));
                  }
                  p = e ? gp.y : gp.x;
                  ds = e ? gd.y : gd.x;
                } else if constexpr (PHI == GDPA_PHI_GELU) {
                  if (e == 0)           // both columns of the pair, in packed arithmetic
                    gelu_fg2(__ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                        make_float2(sc, sc), make_float2(b1k, b1k)),
                             gp, gd);
                  p = e ? gp.y : gp.x;
                  ds = g * (e ? gd.y : gd.x);
                } else {
                  if (e == 0)           // both columns of the pair, in packed arithmetic
                    gp = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                    make_float2(sc, sc), make_float2(b1k, b1k));
                  p = e ? gp.y : gp.x;
                  ds = g;
                }
                // softmax rows past the sample already give P = dS = 0 (-LSE = -inf)
                const bool valid = SOFTMAX || FULL || rbase + r < n;
                pv[e] = valid ? p : 0.f;
                dv2[e] = valid ? ds : 0.f;
                if constexpr (BIAS) db1_acc += dv2[e];
              }
              pp[c / 2] = pack_bf16x2(pv[0], pv[1]);
              dd[c / 2] = pack_bf16x2(dv2[0], dv2[1]);
            }
            tmem_st_x16(tmem + lane_off + C::COL_S + 64 * grp + 16 * ch, pp);
            // dS^T line `lrow` of chunk `grp`, 16-byte pieces 4ch..4ch+3, 128B swizzle
            const uint32_t line = sDS + grp * 16384 + lrow * 128;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
              const uint32_t j = 4 * ch + jj;
              const uint32_t addr = line + ((j ^ (uint32_t)(lrow & 7)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dd[4 * jj]),
                           "r"(dd[4 * jj + 1]), "r"(dd[4 * jj + 2]), "r"(dd[4 * jj + 3])
                           : "memory");
            }
          }
        };
        if (SOFTMAX || rbase + 64 <= n)
          half_body(std::true_type{});
        else
          half_body(std::false_type{});
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL));
        if (!C::DQ2) {
          if (!drain_dq(i, qs)) {
            ok = false;
            break;
          }
        } else if (i > 0 && !drain_dq(i - 1, qs - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && C::DQ2 && !drain_dq(nq - 1, qs - 1)) ok = false;
      if (!ok) break;
      if constexpr (BIAS) add_key_bias_grad(a, it, key, db1_acc);
      // ---------------------------------------------------------- dV / dK of this key block
      bool w = mbar_wait(bar(C::B_ACCFULL), ic & 1u, abort_flag, kTimeoutNs);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      {
        // Group 0 writes dV, group 1 s*dK.  Each lane owns one key row; the
        // warp passes its 32 rows through its own shared-memory area (64
        // columns at a time, 16-byte chunks swizzled by row) so that every
        // global store instruction writes 4 whole 128-byte row pieces.
        const uint32_t src = tmem + lane_off + (grp == 0 ? C::COL_DV : C::COL_DK);
        const float mul = grp == 0 ? 1.f : sc;
        const uint32_t kstg = base + C::OFF_KSTG + (uint32_t)(warp - 4) * C::KSTG_WARP;
        __nv_bfloat16* blk = (grp == 0 ? a.dv : a.dk) +
                             (((int64_t)it.b * a.h + it.head) * a.m + it.row0 + quad * 32) * DH;
        const int rl = lane >> 3, jl = lane & 7;         // read-back: row in group of 4, chunk
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 64) {
          if (lane == 0) bulk_wait_group_read0();      // a dQ reduce may still read the area
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 64; c += 16) {
            uint32_t v[16];
            tmem_ld_x16(src + c0 + c, v);
            tmem_wait_ld();
            if (c0 + c + 16 == DH) {
              tc_fence_before();
              mbar_arrive(bar(C::B_ACCEMPTY));          // the accumulators are free
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              uint32_t pk[4];
#pragma unroll
              for (int u = 0; u < 4; ++u)
                pk[u] = pack_bf16x2(__uint_as_float(v[8 * j + 2 * u]) * mul,
                                    __uint_as_float(v[8 * j + 2 * u + 1]) * mul);
              const uint32_t chunk = (uint32_t)(c / 8 + j);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                           ::"r"(kstg + lane * 128 + ((chunk ^ (uint32_t)(lane & 7)) << 4)),
                           "r"(pk[0]), "r"(pk[1]), "r"(pk[2]), "r"(pk[3])
                           : "memory");
            }
          }
          __syncwarp();
#pragma unroll
          for (int it4 = 0; it4 < 8; ++it4) {
            const int r = it4 * 4 + rl;                  // row within this warp's 32
            uint4 val;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                         : "r"(kstg + r * 128 + (((uint32_t)jl ^ (uint32_t)(r & 7)) << 4)));
            if (it.row0 + quad * 32 + r < a.m)
              *reinterpret_cast<uint4*>(blk + (int64_t)r * DH + c0 + jl * 8) = val;
          }
          __syncwarp();
        }
      }
      ++ic;
    }
    if (lane == 0) bulk_wait_group0();                // reduces done before the CTA exits
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    report(a.ws, GDPA_ERR_TIMEOUT);
    volatile int never = 0;
    if (warp == 1 && lane == 0) {
      mma_commit(bar(C::B_DRAIN));
      mbar_wait(bar(C::B_DRAIN), 0, &never, kTimeoutNs);
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 200000ull) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// ---------------------------------------------------------------- half-tile kernel (dh <= 64)
//
// Same products as above, but each 128-row query tile is processed as two
// 64-row halves with their own S^T/dP^T buffers in TMEM, so that activation
// group h works on half h while the tensor core computes the other half:
//   ST(i,0) ST(i,1) | dVdK(i,0) ST(i+1,0) | dVdK(i,1) dQ(i) ST(i+1,1) | ...
// where ST(i,h) = {S^T, dP^T} of rows 64h..64h+63 of tile i (M = 128 keys,
// N = 64 rows), dVdK(i,h) adds that half's P^T dO and dS^T Q (K = 64 rows),
// and dQ(i) = dS K over the whole tile once both halves of dS^T are written.
// dS^T and dQ are double-buffered by tile parity.
//
// TMEM: S^T_h [128h, 128h+64), dP^T_h [128h+64, 128h+128) (P^T_h aliases the
// first 32 columns of S^T_h), dV [256, 256+dh), dK [256+dh, 256+2dh),
// dQ_c [256+2dh+c*dh, 256+3dh+c*dh).
//
// Schedule:
//   - K/V have two slots, so the producer loads the next item's key block and
//     query tiles while the current item runs, and the MMA thread issues the
//     next item's first S^T/dP^T products right after the current item's dQ;
//   - a fourth warpgroup (warps 12-15, one per TMEM lane quadrant) drains dQ
//     (bulk reduce-add) and dV/dK (bulk store), and warp 2 loads the softmax
//     row statistics one tile ahead, so the two activation groups only form
//     P^T and dS^T.
// Each drain warp reduces the dQ of its own 32 rows through a 4 KB staging box
// of its own, one column half at a time, and skips rows that all lie past the
// sample.  An item's dV/dK are staged in its last tile's dS^T buffer (whose
// readers are all in the completed products).  Before the MMA thread issues
// the S^T products of the tile that will overwrite a dS^T buffer (two tiles
// later), it waits on STGFREE of that buffer: the drain group arrives on it as
// soon as the tile's dQ products complete, or, at an item's last tile, once
// the dV/dK stores have read the buffer.
// Registers (512 threads at 128 each): warps 0-3 drop to 72, the drain group
// to 104, the activation groups rise to 168 (4 x 128 x (72+104+168+168) = 65536).
constexpr int kHalfThreads = 512;

template <int DH>
struct BwdHalfCfg {
  static_assert(DH <= 64, "half-tile pipeline needs dh <= 64");
  static constexpr uint32_t ROWB = DH * 2;
  static constexpr uint32_t TILEB = 128 * ROWB;            // [128 x DH] bf16
  static constexpr uint32_t SW = DH < 64 ? kSw64 : kSw128;
  static constexpr uint32_t ATOM = 8 * ROWB;
  static constexpr int NSTG = 2, NKV = 2;
  static constexpr uint32_t DSB = 2 * 128 * 128;           // one dS^T buffer, two 16 KB halves
  static constexpr uint32_t COL_DV = 256, COL_DK = 256 + DH, COL_DQ = 256 + 2 * DH;
  // dV/dK staging rows: DH bf16
  static constexpr uint32_t SROWB = 2 * DH;
  static constexpr int B_KVFULL = 0, B_KVEMPTY = 2, B_SFULL = 4, B_PFULL = 6, B_DQFULL = 8,
                       B_DQEMPTY = 10, B_ACCFULL = 12, B_ACCEMPTY = 13, B_DRAIN = 14,
                       B_DSYNC = 15, B_STGFREE = 16, B_STFULL = 18, B_STEMPTY = 18 + NSTG,
                       B_STATFULL = 18 + 2 * NSTG, B_STATEMPTY = 20 + 2 * NSTG,
                       NBAR = 22 + 2 * NSTG;
  static constexpr uint32_t OFF_KV = 0;                    // slot s: K at 2s TILEB, V at (2s+1) TILEB
  static constexpr uint32_t OFF_STG = NKV * 2 * TILEB;
  static constexpr uint32_t OFF_DS = OFF_STG + NSTG * 2 * TILEB;
  static constexpr uint32_t OFF_CTL = OFF_DS + 2 * DSB;
  // + a two-slot ring of row statistics: [slot][log2-scaled LSE, D][128 rows] fp32
  static constexpr uint32_t CTL_BYTES = 1024 + 2 * 2 * 128 * 4;
  // + one dQ staging box per drain warp: its 32 rows x DH/2 fp32 (a column half)
  static constexpr uint32_t DQSB = 32 * 2 * DH;
  static constexpr uint32_t OFF_DQS = (OFF_CTL + CTL_BYTES + 1023u) & ~1023u;
  static constexpr uint32_t SMEM_USED = 1024 + OFF_DQS + 4 * DQSB;
  static constexpr uint32_t SMEM = SMEM_USED > 120u * 1024u ? SMEM_USED : 120u * 1024u;
  static_assert(SMEM <= 232448u, "exceeds the 227 KB of shared memory a CTA can have");
  static_assert(COL_DQ + 2 * DH <= 512, "TMEM columns");
  static_assert(128 * SROWB <= DSB / 2, "a staging box fits in a dS^T half");
  static_assert(OFF_STG % 1024 == 0 && OFF_DS % 1024 == 0 && OFF_DQS % 1024 == 0 &&
                DQSB % 1024 == 0, "swizzle atoms need 1024-B alignment");
  static_assert(8 * NBAR + 8 <= 1024, "barriers, TMEM slot and abort flag share the first 1 KB");
};

// 16-byte chunk j of staging row r, swizzled like the bulk copies' maps
// (128 B rows: 128B swizzle, 64 B rows: 64B swizzle)
template <int DH>
__device__ __forceinline__ uint32_t stage_chunk(uint32_t box, int r, int j) {
  const int sw = DH == 64 ? (r & 7) : ((r >> 1) & 3);
  return box + (uint32_t)(r * 2 * DH) + ((uint32_t)(j ^ sw) << 4);
}

// Modes of the half kernel: GDPA (keys and values per sample [B, h, m, dh]),
// seed-query pooling (the seeds [h, S, dh] are the one query tile of every
// item; keys and values are the jagged tokens) and the causal sliding window
// (queries, keys and values are the jagged tokens; an item visits only the
// query tiles whose window reaches its key block).
constexpr int kModeGdpa = 0, kModePool = 1, kModeWindow = 2;

template <int DH, int PHI, bool BIAS, int MODE>
__global__ void __launch_bounds__(kHalfThreads, 1)
gdpa_bwd_half_kernel(const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmG,
                   const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV,
                   const __grid_constant__ CUtensorMap tmDQ,
                   const __grid_constant__ CUtensorMap tmDV,
                   const __grid_constant__ CUtensorMap tmDK, const BwdArgs a) {
  using C = BwdHalfCfg<DH>;
  constexpr bool SOFTMAX = PHI == GDPA_PHI_SOFTMAX;
  constexpr bool POOL = MODE == kModePool, WIN = MODE == kModeWindow, JAG = MODE != kModeGdpa;
  static_assert(!JAG || (SOFTMAX && !BIAS), "pooling and the window are softmax attention");
  constexpr uint32_t IDESC_T = idesc_bf16(128, 64, 0, 0);    // S^T, dP^T of a half: N = 64 rows
  constexpr uint32_t IDESC_KV = idesc_bf16(128, DH, 0, 1);   // dV, dK (B MN-major)
  constexpr uint32_t IDESC_Q = idesc_bf16(128, DH, 1, 1);    // dQ (A and B MN-major)

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sKV = base + C::OFF_KV, sStg = base + C::OFF_STG, sDS = base + C::OFF_DS;
  const uint32_t sDQS = base + C::OFF_DQS;
  uint8_t* ctl = gbase + C::OFF_CTL;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * C::NBAR + 4);
  float* stats = reinterpret_cast<float*>(ctl + 1024);   // [2 slots][-LSE, -D][128]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_KVFULL + i), 1);
      mbar_init(bar(C::B_KVEMPTY + i), 1);
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 128);
      mbar_init(bar(C::B_DQFULL + i), 1);
      mbar_init(bar(C::B_DQEMPTY + i), 128);
      mbar_init(bar(C::B_STGFREE + i), 1);
      mbar_init(bar(C::B_STATFULL + i), 1);
      mbar_init(bar(C::B_STATEMPTY + i), 8);       // lane 0 of each activation warp
    }
    mbar_init(bar(C::B_ACCFULL), 1);
    mbar_init(bar(C::B_ACCEMPTY), 128);
    mbar_init(bar(C::B_DRAIN), 1);
    mbar_init(bar(C::B_DSYNC), 128);
    for (int i = 0; i < C::NSTG; ++i) {
      mbar_init(bar(C::B_STFULL + i), 1);
      mbar_init(bar(C::B_STEMPTY + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmG);
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    prefetch_tmap(&tmDQ);
    prefetch_tmap(&tmDV);
    prefetch_tmap(&tmDK);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int count = a.ws->status == GDPA_ERR_INVALID_ARG ? 0 : a.ws->tile_count;
  const int wg = warp >> 2;
  auto next_item = [&](int t) -> int {            // next item of this CTA with query rows
    while (t < count && a.tiles[t].rows == 0) t += gridDim.x;
    return t;
  };
  // query tiles of an item: the first (fi, in 128-row tiles of the sample)
  // and the count.  GDPA: all of the sample's tiles; pooling: the seed tile;
  // window: the tiles whose rows t satisfy row0 <= t < row0 + 128 + window - 1.
  auto tiles_of = [&](const Tile& it, int& fi) -> int {
    if constexpr (POOL) {
      fi = 0;
      return 1;
    } else if constexpr (WIN) {
      fi = it.row0 >> 7;
      const int last = min(it.rows - 1, it.row0 + 127 + a.window - 1);
      return (last >> 7) - fi + 1;
    } else {
      fi = 0;
      return (it.rows + 127) >> 7;
    }
  };

  if (wg == 0) {
    setmaxnreg_dec<72>();
    if (warp == 0 && lane == 0) {
      // -------------------------------------------------------- producer
      // runs up to one item ahead: K/V of the next item go to the other slot
      uint32_t kvi = 0, stage = 0, sphase = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < count; t += gridDim.x) {
        const Tile it = a.tiles[t];
        if (it.rows == 0) continue;
        int fi;
        const int nq = tiles_of(it, fi);
        const int t0 = a.offsets[it.b];
        const uint32_t slot = kvi & 1u;
        if (!mbar_wait(bar(C::B_KVEMPTY + slot), ((kvi >> 1) & 1u) ^ 1u, abort_flag, kTimeoutNs))
          break;
        const uint32_t sK = sKV + slot * 2 * C::TILEB;
        mbar_expect_tx(bar(C::B_KVFULL + slot), 2 * C::TILEB);
        if constexpr (JAG) {          // tokens [T, h, DH]: rows past the sample are masked later
          tma_load_3d(sK, &tmK, bar(C::B_KVFULL + slot), 0, it.head, t0 + it.row0);
          tma_load_3d(sK + C::TILEB, &tmV, bar(C::B_KVFULL + slot), 0, it.head, t0 + it.row0);
        } else {
          tma_load_4d(sK, &tmK, bar(C::B_KVFULL + slot), 0, it.row0, it.head, it.b);
          tma_load_4d(sK + C::TILEB, &tmV, bar(C::B_KVFULL + slot), 0, it.row0, it.head, it.b);
        }
        for (int i = 0; i < nq; ++i) {
          if (!mbar_wait(bar(C::B_STEMPTY + stage), sphase ^ 1u, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          const uint32_t dst = sStg + stage * 2 * C::TILEB;
          mbar_expect_tx(bar(C::B_STFULL + stage), 2 * C::TILEB);
          if constexpr (POOL) {       // seeds [h, S, DH], dO [B*h, S, DH]; rows >= S read as zero
            tma_load_3d(dst, &tmQ, bar(C::B_STFULL + stage), 0, 0, it.head);
            tma_load_3d(dst + C::TILEB, &tmG, bar(C::B_STFULL + stage), 0, 0,
                        it.b * a.h + it.head);
          } else {
            tma_load_3d(dst, &tmQ, bar(C::B_STFULL + stage), 0, it.head, t0 + 128 * (fi + i));
            tma_load_3d(dst + C::TILEB, &tmG, bar(C::B_STFULL + stage), 0, it.head,
                        t0 + 128 * (fi + i));
          }
          if (++stage == (uint32_t)C::NSTG) {
            stage = 0;
            sphase ^= 1u;
          }
        }
        ++kvi;
      }
    } else if (warp == 1 && lane == 0) {
      // -------------------------------------------------------- MMA issuer
      uint32_t stage = 0, sphase = 0, qs = 0, kvi = 0;
      bool ok = true;
      // slot 0's descriptors; slot s starts s * 2 * TILEB bytes further
      const uint64_t dk0 = smem_desc(sKV, 16, C::ATOM, C::SW);                 // K, K-major (S^T)
      const uint64_t dv0 = smem_desc(sKV + C::TILEB, 16, C::ATOM, C::SW);      // V, K-major (dP^T)
      const uint64_t kmn0 = smem_desc(sKV, C::TILEB, C::ATOM, C::SW);          // K, MN-major (dQ)
      auto wait_bar = [&](int which, uint32_t ph) -> bool {
        if (!mbar_wait(bar(which), ph, abort_flag, kTimeoutNs)) return false;
        tc_fence_after();
        return true;
      };
      // ST(q, h): S^T_h = K Q[64h..]^T and dP^T_h = V dO[64h..]^T of tile q, in stage `st`.
      // Before half 0, the drain group must be done with tile q-2's staging in
      // the dS^T buffer that tile q's activation will write.
      auto issue_st = [&](uint32_t q, uint32_t st, int h, uint32_t slot) -> bool {
        if (h == 0 && !wait_bar(C::B_STGFREE + (int)(q & 1u), ((q >> 1) & 1u) ^ 1u)) return false;
        const uint32_t qaddr = sStg + st * 2 * C::TILEB + 64 * h * C::ROWB;
        const uint64_t q0 = smem_desc(qaddr, 16, C::ATOM, C::SW);
        const uint64_t g0 = smem_desc(qaddr + C::TILEB, 16, C::ATOM, C::SW);
        const uint64_t dk = desc_advance(dk0, slot * 2 * C::TILEB);
        const uint64_t dv = desc_advance(dv0, slot * 2 * C::TILEB);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k)
          mma_ss(tmem + 128 * h, desc_advance(dk, k * 32), desc_advance(q0, k * 32), IDESC_T,
                 k > 0 ? 1u : 0u);
#pragma unroll
        for (int k = 0; k < DH / 16; ++k)
          mma_ss(tmem + 128 * h + 64, desc_advance(dv, k * 32), desc_advance(g0, k * 32), IDESC_T,
                 k > 0 ? 1u : 0u);
        mma_commit(bar(C::B_SFULL + h));
        return true;
      };
      // dVdK(h): dV += P^T_h dO[64h..], dK += dS^T[64h..] Q[64h..] of the tile in `st`
      auto issue_dvdk = [&](uint32_t st, int h, uint32_t c, bool first) {
        const uint32_t qaddr = sStg + st * 2 * C::TILEB + 64 * h * C::ROWB;
        const uint64_t gmn = smem_desc(qaddr + C::TILEB, C::TILEB, C::ATOM, C::SW);   // dO, MN-major
        const uint64_t qmn = smem_desc(qaddr, C::TILEB, C::ATOM, C::SW);              // Q, MN-major
        // both A operands from TMEM (P^T_h over S^T_h's first columns, dS^T_h over
        // dP^T_h's): only the 2 KB B tiles come from shared memory, whose
        // bandwidth N = 64 products are short of
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ts(tmem + C::COL_DV, tmem + 128 * h + 8 * k, desc_advance(gmn, k * 2 * C::ATOM),
                 IDESC_KV, (first && k == 0) ? 0u : 1u);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ts(tmem + C::COL_DK, tmem + 128 * h + 64 + 8 * k, desc_advance(qmn, k * 2 * C::ATOM),
                 IDESC_KV, (first && k == 0) ? 0u : 1u);
      };
      // One pass over every (item, query tile) of this CTA.
      int t = next_item(blockIdx.x);
      int fi_unused;
      if (t < count) {
        int nq = tiles_of(a.tiles[t], fi_unused);
        uint32_t slot = 0;
        ok = wait_bar(C::B_KVFULL + 0, 0) && wait_bar(C::B_STFULL + stage, sphase) &&
             issue_st(0, stage, 0, slot) && issue_st(0, stage, 1, slot);
        for (int i = 0; ok;) {
          const uint32_t c = qs & 1u;
          const bool last = i + 1 == nq;
          const int tn = last ? next_item(t + gridDim.x) : t;
          const bool has_next = tn < count;
          const uint32_t nslot = last ? slot ^ 1u : slot;
          const uint32_t nkvi = last ? kvi + 1 : kvi;
          uint32_t nst = stage + 1, nph = sphase;
          if (nst == (uint32_t)C::NSTG) {
            nst = 0;
            nph ^= 1u;
          }
          // half 0 of this tile, then (within an item) the next tile's half-0 products
          if (!wait_bar(C::B_PFULL + 0, c) ||
              (i == 0 && !wait_bar(C::B_ACCEMPTY, (kvi & 1u) ^ 1u))) {
            ok = false;
            break;
          }
          issue_dvdk(stage, 0, c, i == 0);
          if (has_next && !last) {
            if (!wait_bar(C::B_STFULL + nst, nph) || !issue_st(qs + 1, nst, 0, nslot)) {
              ok = false;
              break;
            }
          }
          // half 1 and the tile's dQ
          if (!wait_bar(C::B_PFULL + 1, c)) {
            ok = false;
            break;
          }
          issue_dvdk(stage, 1, c, false);
          mma_commit(bar(C::B_STEMPTY + stage));
          if (!wait_bar(C::B_DQEMPTY + c, ((qs >> 1) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          {
            const uint64_t dsm = smem_desc(sDS + c * C::DSB, 16384, 1024, kSw128);   // dS, MN-major
            const uint64_t kmn = desc_advance(kmn0, slot * 2 * C::TILEB);
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_ss(tmem + C::COL_DQ + c * DH, desc_advance(dsm, k * 2048),
                     desc_advance(kmn, k * 2 * C::ATOM), IDESC_Q, k > 0 ? 1u : 0u);
            mma_commit(bar(C::B_DQFULL + c));
          }
          if (last) {
            mma_commit(bar(C::B_KVEMPTY + slot));
            mma_commit(bar(C::B_ACCFULL));
            // the next item's first products, once this item's are all issued
            if (has_next &&
                (!wait_bar(C::B_KVFULL + nslot, (nkvi >> 1) & 1u) ||
                 !wait_bar(C::B_STFULL + nst, nph) || !issue_st(qs + 1, nst, 0, nslot))) {
              ok = false;
              break;
            }
          }
          if (has_next && !issue_st(qs + 1, nst, 1, nslot)) {
            ok = false;
            break;
          }
          stage = nst;
          sphase = nph;
          ++qs;
          if (!has_next) break;
          if (last) {
            t = tn;
            nq = tiles_of(a.tiles[t], fi_unused);
            slot = nslot;
            kvi = nkvi;
            i = 0;
          } else {
            ++i;
          }
        }
      }
    }
    else if (warp == 2 && SOFTMAX) {
      // -------------------------------------------------------- row statistics
      // -LSE (log2-scaled) and -D of each query tile into the ring, one tile ahead
      uint32_t q = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < count; t += gridDim.x) {
        const Tile it = a.tiles[t];
        if (it.rows == 0) continue;
        int fi;
        const int nq = tiles_of(it, fi);
        const int t0 = a.offsets[it.b];
        for (int i = 0; i < nq; ++i, ++q) {
          const uint32_t slot = q & 1u;
          const bool w = mbar_wait(bar(C::B_STATEMPTY + (int)slot), ((q >> 1) & 1u) ^ 1u,
                                   abort_flag, kTimeoutNs);
          if (!__all_sync(0xffffffffu, w)) {
            ok = false;
            break;
          }
          float* ring = stats + slot * 256;      // negated, as the activation adds them
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int r = 32 * u + lane, rg = 128 * (fi + i) + r;
            // rows past the sample (pooling: seeds >= S) take -LSE = -inf, so
            // that their P and dS come out exactly 0
            float l = INFINITY, d = 0.f;
            if (POOL ? r < a.S : rg < it.rows) {
              const int64_t at = POOL ? ((int64_t)it.b * a.h + it.head) * a.S + r
                                      : (int64_t)it.head * a.T + t0 + rg;
              l = __ldg(a.lse + at) * 1.4426950408889634f;
              d = __ldg(a.dsum + at);
            }
            ring[r] = -l;
            ring[128 + r] = -d;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::B_STATFULL + (int)slot));
        }
      }
    }
  } else if (wg <= 2) {
    // ---------------------------------------------------------- activation groups
    setmaxnreg_inc<168>();
    const int grp = wg - 1;                            // the 64-row half this group owns
    const int quad = warp & 3;
    const int lrow = quad * 32 + lane;                 // TMEM lane: key
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float c2 = a.scale_log2, sc = a.scale, half_sc = 0.5f * a.scale;
    uint32_t qs = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < count; t += gridDim.x) {
      const Tile it = a.tiles[t];
      const int n = it.rows;
      if (n == 0) continue;
      int fi;
      const int nq = tiles_of(it, fi);
      // biased variant: this key's bias (log2 units for softmax, halved for
      // SiLU) and this thread's sum of dS over its half of the tokens (for db1)
      const int key = it.row0 + lrow;
      const bool key_ok = !JAG || key < n;              // jagged keys: rows past the sample
      const float b1k = BIAS ? key_bias(a, it, key) : 0.f;
      const float b1l = b1k * 1.4426950408889634f, hb = 0.5f * b1k;
      // added to the softmax exponent of every pair of this key (log2 units)
      const float kterm = BIAS ? b1l : (key_ok ? 0.f : -INFINITY);
      float db1_acc = 0.f;
      for (int i = 0; i < nq; ++i, ++qs) {
        const int rbase = 128 * (fi + i) + 64 * grp;   // first sample row (seed) of this half
        const int band0 = rbase - key;                 // window: row rbase + r is in band iff
                                                       // 0 <= band0 + r < window
        const uint32_t dsb = sDS + (qs & 1u) * C::DSB + grp * 16384;
        const float* st_l = stats + (qs & 1u) * 256 + 64 * grp;
        const float* st_d = st_l + 128;
        bool w = mbar_wait(bar(C::B_SFULL + grp), qs & 1u, abort_flag, kTimeoutNs);
        if constexpr (SOFTMAX)
          w = w && mbar_wait(bar(C::B_STATFULL + (int)(qs & 1u)), (qs >> 1) & 1u, abort_flag,
                             kTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // every query row (seed) of this half lies past the sample: its P^T and
        // dS^T columns are zero, and the dQ rows it would feed are never added
        const bool empty_half = rbase >= (POOL ? a.S : n);
        if (empty_half) {
          uint32_t z[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) z[u] = 0u;
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            tmem_st_x16(tmem + lane_off + 128 * grp + 16 * ch, z);
            tmem_st_x16(tmem + lane_off + 128 * grp + 64 + 16 * ch, z);
          }
        } else {
          // FULL: every query row of the half lies in the sample, so the
          // activations other than softmax need no row mask either
          auto half_body = [&](auto full_tag) {
            constexpr bool FULL = decltype(full_tag)::value;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
              uint32_t s[32], dp[32];
              tmem_ld_x32(tmem + lane_off + 128 * grp + 32 * ch, s);
              tmem_ld_x32(tmem + lane_off + 128 * grp + 64 + 32 * ch, dp);
              tmem_wait_ld();
              uint32_t pp[16], dd[16];
              [[maybe_unused]] float4 nl4, nd4;   // softmax: -LSE and -D of rows c..c+3
#pragma unroll
              for (int c = 0; c < 32; c += 2) {
                float pv[2], dv2[2];
                [[maybe_unused]] float2 gp, gd;   // P and dS (GELU: phi') of the pair
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                  const int r = 32 * ch + c + e;
                  const float x = __uint_as_float(s[c + e]);
                  const float g = __uint_as_float(dp[c + e]);
                  float p, ds;
                  // u = s x + b1 (the biased logit; b1k = 0 without a key bias)
                  if constexpr (SOFTMAX) {
                    if (e == 0) {         // both columns of the pair, in packed arithmetic
                      if ((c & 2) == 0) {   // rows r..r+3 (16-byte aligned)
                        nl4 = *reinterpret_cast<const float4*>(st_l + r);
                        nd4 = *reinterpret_cast<const float4*>(st_d + r);
                      }
                      const float2 nl = (c & 2) ? make_float2(nl4.z, nl4.w) : make_float2(nl4.x, nl4.y);
                      const float2 nd = (c & 2) ? make_float2(nd4.z, nd4.w) : make_float2(nd4.x, nd4.y);
                      // the key's term: its bias, or -inf for a jagged key past the sample
                      float2 u = __ffma2_rn(
                          make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                          make_float2(c2, c2),
                          BIAS || JAG ? __fadd2_rn(nl, make_float2(kterm, kterm)) : nl);
                      if constexpr (WIN) {    // the band key <= t < key + window
                        u.x = (uint32_t)(band0 + r) < (uint32_t)a.window ? u.x : -INFINITY;
                        u.y = (uint32_t)(band0 + r + 1) < (uint32_t)a.window ? u.y : -INFINITY;
                      }
                      gp = make_float2(ex2_approx(u.x), ex2_approx(u.y));
                      gd = __fmul2_rn(gp, __fadd2_rn(make_float2(__uint_as_float(dp[c]),
                                                                 __uint_as_float(dp[c + 1])),
                                                     nd));
                    }
                    p = e ? gp.y : gp.x;
                    ds = e ? gd.y : gd.x;
                  } else if constexpr (PHI == GDPA_PHI_SILU) {
                    if (e == 0)           // both columns of the pair, in packed arithmetic
                      silu_fg2(__ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                          make_float2(half_sc, half_sc), make_float2(hb, hb)),
                               make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])), gp, gd);
                    p = e ? gp.y : gp.x;
                    ds = e ? gd.y : gd.x;
                  } else if constexpr (PHI == GDPA_PHI_RELU) {
                    if (e == 0) {         // both columns of the pair, in packed arithmetic
                      const float2 u = __ffma2_rn(
                          make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                          make_float2(sc, sc), make_float2(b1k, b1k));
                      gp = make_float2(relu_f(u.x), relu_f(u.y));
                      gd = __fmul2_rn(make_float2(__uint_as_float(dp[c]), __uint_as_float(dp[c + 1])),
                                      make_float2(relu_grad(u.x), relu_grad(u.y)));
                    }
                    p = e ? gp.y : gp.x;
                    ds = e ? gd.y : gd.x;
                  } else if constexpr (PHI == GDPA_PHI_GELU) {
                    if (e == 0)           // both columns of the pair, in packed arithmetic
                      gelu_fg2(__ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                          make_float2(sc, sc), make_float2(b1k, b1k)),
                               gp, gd);
                    p = e ? gp.y : gp.x;
                    ds = g * (e ? gd.y : gd.x);
                  } else {
                    if (e == 0)           // both columns of the pair, in packed arithmetic
                      gp = __ffma2_rn(make_float2(__uint_as_float(s[c]), __uint_as_float(s[c + 1])),
                                      make_float2(sc, sc), make_float2(b1k, b1k));
                    p = e ? gp.y : gp.x;
                    ds = g;
                  }
                  // softmax: rows past the sample (-LSE = -inf), keys past it and
                  // pairs outside the window (exponent -inf) give P = dS = 0 exactly
                  const bool valid = SOFTMAX || FULL || rbase + r < n;
                  pv[e] = valid ? p : 0.f;
                  dv2[e] = valid ? ds : 0.f;
                  if constexpr (BIAS) db1_acc += dv2[e];
                }
                pp[c / 2] = pack_bf16x2(pv[0], pv[1]);
                dd[c / 2] = pack_bf16x2(dv2[0], dv2[1]);
              }
              tmem_st_x16(tmem + lane_off + 128 * grp + 16 * ch, pp);
              // dS^T_h as bf16 over dP^T_h's first 32 columns (read above) for the dK product
              tmem_st_x16(tmem + lane_off + 128 * grp + 64 + 16 * ch, dd);
              // dS^T line `lrow` of this half's chunk, 16-byte pieces 4ch..4ch+3, 128B swizzle
              const uint32_t line = dsb + lrow * 128;
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                const uint32_t j = 4 * ch + jj;
                const uint32_t addr = line + ((j ^ (uint32_t)(lrow & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dd[4 * jj]),
                             "r"(dd[4 * jj + 1]), "r"(dd[4 * jj + 2]), "r"(dd[4 * jj + 3])
                             : "memory");
              }
            }
          };
          if (SOFTMAX || rbase + 64 <= n)
            half_body(std::true_type{});
          else
            half_body(std::false_type{});
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + grp));
        if constexpr (SOFTMAX) {
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(C::B_STATEMPTY + (int)(qs & 1u)));
        }
      }
      if constexpr (BIAS) {
        if (ok) add_key_bias_grad(a, it, key, db1_acc);
      }
    }
  } else {
    // ---------------------------------------------------------- drain group
    setmaxnreg_dec<104>();
    const int quad = warp & 3;
    const int lrow = quad * 32 + lane;                 // TMEM lane: query row (dQ) or key (dV, dK)
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const float sc = a.scale;
    uint32_t qs = 0, ic = 0, sync_phase = 0;
    bool ok = true;
    auto group_sync = [&]() -> bool {                 // the 128 threads of this group
      mbar_arrive(bar(C::B_DSYNC));
      const bool w = mbar_wait(bar(C::B_DSYNC), sync_phase, abort_flag, kTimeoutNs);
      sync_phase ^= 1u;
      return __all_sync(0xffffffffu, w);
    };
    // one key row of DH columns from 16-column TMEM loads, as bf16 times `mul`
    // (dV, dK), into 16-byte chunks of a staging box
    auto stage_bf16 = [&](uint32_t src, uint32_t box, float mul) {
#pragma unroll
      for (int c = 0; c < DH; c += 16) {
        uint32_t v[16];
        tmem_ld_x16(src + c, v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          uint32_t pk[4];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            pk[u] = pack_bf16x2(__uint_as_float(v[8 * j + 2 * u]) * mul,
                                __uint_as_float(v[8 * j + 2 * u + 1]) * mul);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                       ::"r"(stage_chunk<DH>(box, lrow, c / 8 + j)), "r"(pk[0]), "r"(pk[1]),
                       "r"(pk[2]), "r"(pk[3])
                       : "memory");
        }
      }
    };
    // one key row of DH columns from TMEM, times `mul`, as bf16 straight to
    // global memory at dst (NULL: read only; every lane takes part in the loads)
    auto store_row = [&](uint32_t src, __nv_bfloat16* dst, float mul) {
#pragma unroll
      for (int c = 0; c < DH; c += 16) {
        uint32_t v[16];
        tmem_ld_x16(src + c, v);
        tmem_wait_ld();
        uint32_t pk[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          pk[u] = pack_bf16x2(__uint_as_float(v[2 * u]) * mul, __uint_as_float(v[2 * u + 1]) * mul);
        if (dst) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + c);
          d4[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          d4[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        }
      }
    };
    for (int t = blockIdx.x; ok && t < count; t += gridDim.x) {
      const Tile it = a.tiles[t];
      const int n = it.rows;
      if (n == 0) {                                    // no tokens: dK = dV = 0
        const int key = it.row0 + lrow;
        if (key < a.m) {
          const int64_t row = (((int64_t)it.b * a.h + it.head) * a.m + key) * DH;
          uint4* v4 = reinterpret_cast<uint4*>(a.dv + row);
          uint4* k4 = reinterpret_cast<uint4*>(a.dk + row);
#pragma unroll
          for (int c = 0; c < DH / 8; ++c) {
            v4[c] = make_uint4(0u, 0u, 0u, 0u);
            k4[c] = make_uint4(0u, 0u, 0u, 0u);
          }
        }
        continue;
      }
      int fi;
      const int nq = tiles_of(it, fi);
      const int t0 = a.offsets[it.b];
      for (int i = 0; i < nq; ++i, ++qs) {
        const uint32_t b = qs & 1u;
        // dQ of tile qs: the tile's products are complete
        bool w = mbar_wait(bar(C::B_DQFULL + (int)b), (qs >> 1) & 1u, abort_flag, kTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t stg = sDS + b * C::DSB;
        // within an item the tile's dS^T buffer has no readers left
        if (i + 1 < nq && lrow == 0) mbar_arrive(bar(C::B_STGFREE + (int)b));
        {
          // Each warp reduces its own 32 rows into the fp32 accumulator, one
          // column half at a time through its staging box.  Rows past the
          // sample (pooling: past the seeds) are exact zeros, since their dS
          // entries are zero: a warp whose rows all lie there adds nothing, and
          // rows past T are clipped by the map.
          const int rows_here = POOL ? a.S : n - 128 * (fi + i);
          const bool adds = quad * 32 < rows_here;
          const uint32_t box = sDQS + quad * C::DQSB;
          const uint32_t src = tmem + lane_off + C::COL_DQ + b * DH;
#pragma unroll
          for (int hc = 0; hc < 2; ++hc) {
            uint32_t v[DH / 2];
#pragma unroll
            for (int c = 0; c < DH / 2; c += 16)
              tmem_ld_x16(src + hc * (DH / 2) + c, *reinterpret_cast<uint32_t(*)[16]>(&v[c]));
            tmem_wait_ld();
            if (hc == 1) {
              tc_fence_before();
              mbar_arrive(bar(C::B_DQEMPTY + (int)b));
            }
            if (adds) {
              if (lane == 0) bulk_wait_group_read0();   // the box's previous reduce has read it
              __syncwarp();
#pragma unroll
              for (int j = 0; j < DH / 8; ++j)
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                             ::"r"(stage_chunk<DH>(box, lane, j)), "r"(v[4 * j]),
                             "r"(v[4 * j + 1]), "r"(v[4 * j + 2]), "r"(v[4 * j + 3])
                             : "memory");
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                if constexpr (POOL)   // dseeds [h, S, DH]
                  tma_reduce_add_3d(&tmDQ, box, hc * (DH / 2), 32 * quad, it.head);
                else
                  tma_reduce_add_3d(&tmDQ, box, hc * (DH / 2), it.head,
                                    t0 + 128 * (fi + i) + 32 * quad);
                bulk_commit_group();
              }
            }
          }
        }
        if (i + 1 == nq) {
          // dV and s*dK of this key block, staged in the tile's dS^T buffer
          // (all of its readers are in the completed products)
          w = mbar_wait(bar(C::B_ACCFULL), ic & 1u, abort_flag, kTimeoutNs);
          if (!__all_sync(0xffffffffu, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (JAG && it.row0 + 128 > n) {
            // the key block ends inside the next sample's tokens: each thread
            // writes its own key row when it belongs to this sample
            const int64_t row = ((int64_t)(t0 + it.row0 + lrow) * a.h + it.head) * DH;
            const bool mine = it.row0 + lrow < n;
            store_row(tmem + lane_off + C::COL_DV, mine ? a.dv + row : nullptr, 1.f);
            store_row(tmem + lane_off + C::COL_DK, mine ? a.dk + row : nullptr, sc);
            tc_fence_before();
            mbar_arrive(bar(C::B_ACCEMPTY));
            ++ic;
          } else {
          if (lrow == 0) bulk_wait_group_read0();
          if (!group_sync()) {
            ok = false;
            break;
          }
          stage_bf16(tmem + lane_off + C::COL_DV, stg, 1.f);
          stage_bf16(tmem + lane_off + C::COL_DK, stg + 16384, sc);
          tc_fence_before();
          mbar_arrive(bar(C::B_ACCEMPTY));
          fence_proxy_async_smem();
          if (!group_sync()) {
            ok = false;
            break;
          }
          if (lrow == 0) {
            if constexpr (JAG) {      // dV, dK [T, h, DH]: the whole block is this sample's
              tma_store_3d(&tmDV, stg, 0, it.head, t0 + it.row0);
              tma_store_3d(&tmDK, stg + 16384, 0, it.head, t0 + it.row0);
            } else {
              tma_store_4d(&tmDV, stg, 0, it.row0, it.head, it.b);
              tma_store_4d(&tmDK, stg + 16384, 0, it.row0, it.head, it.b);
            }
            bulk_commit_group();
          }
          ++ic;
          }
        }
        if (i + 1 == nq && lrow == 0) {                // the staging area may be rewritten
          bulk_wait_group_read0();
          mbar_arrive(bar(C::B_STGFREE + (int)b));
        }
      }
    }
    if (lane == 0) bulk_wait_group0();                // copies done before the CTA exits
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    report(a.ws, GDPA_ERR_TIMEOUT);
    volatile int never = 0;
    if (warp == 1 && lane == 0) {
      mma_commit(bar(C::B_DRAIN));
      mbar_wait(bar(C::B_DRAIN), 0, &never, kTimeoutNs);
    }
    if (warp == 0 && lane == 0) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 200000ull) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 2) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side

template <int DH>
bool make_bwd_maps(const gdpa_problem_t& p, const void* q, const void* g, const void* k,
                   const void* v, CUtensorMap* mq, CUtensorMap* mg, CUtensorMap* mk,
                   CUtensorMap* mv) {
  constexpr int CH = DH < 64 ? DH : 64;                 // columns of one swizzled box row
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const CUtensorMapSwizzle sw = DH < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const cuuint64_t qd[3] = {(cuuint64_t)DH, (cuuint64_t)p.h,
                            (cuuint64_t)(p.total_tokens > 0 ? p.total_tokens : 1)};
  const cuuint64_t qs[2] = {(cuuint64_t)DH * 2, (cuuint64_t)p.h * DH * 2};
  const cuuint32_t qb[3] = {(cuuint32_t)CH, 1, 128};
  for (int i = 0; i < 2; ++i)
    if (enc(i ? mg : mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(i ? g : q), qd, qs,
            qb, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  const cuuint64_t kd[4] = {(cuuint64_t)DH, (cuuint64_t)p.m, (cuuint64_t)p.h, (cuuint64_t)p.B};
  const cuuint64_t ks[3] = {(cuuint64_t)DH * 2, (cuuint64_t)p.m * DH * 2,
                            (cuuint64_t)p.h * p.m * DH * 2};
  const cuuint32_t kb[4] = {(cuuint32_t)CH, 128, 1, 1};
  for (int i = 0; i < 2; ++i)
    if (enc(i ? mv : mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(i ? v : k), kd, ks,
            kb, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  return true;
}

// The fp32 dQ accumulator [T, h, DH] as the target of the bulk reduces: boxes
// of 32 rows (one warp's rows) of one head, DH/2 columns (dh <= 64) or 32
// (dh = 128: at most 128 B of a row under the swizzle).
template <int DH>
bool make_dq_map(const gdpa_problem_t& p, float* dq_acc, CUtensorMap* m) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  constexpr int BX = DH / 2 > 32 ? 32 : DH / 2;
  const CUtensorMapSwizzle sw = BX * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  const cuuint32_t estr[3] = {1, 1, 1};
  const cuuint64_t d[3] = {(cuuint64_t)DH, (cuuint64_t)p.h,
                           (cuuint64_t)(p.total_tokens > 0 ? p.total_tokens : 1)};
  const cuuint64_t str[2] = {(cuuint64_t)DH * 4, (cuuint64_t)p.h * DH * 4};
  const cuuint32_t box[3] = {(cuuint32_t)BX, 1, 32};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dq_acc, d, str, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DH, int PHI, bool BIAS>
cudaError_t launch_bwd_t(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                         const void* k, const void* v, const Bias& bs, const float* lse,
                         const float* dsum, const void* g, void* dk, void* dv, float* dq_acc,
                         WsHeader* ws, const Tile* tiles, cudaStream_t st) {
  CUtensorMap mq, mg, mk, mv;
  if (p.total_tokens == 0) q = g = k;   // no query rows: the maps are never read
  if (!make_bwd_maps<DH>(p, q, g, k, v, &mq, &mg, &mk, &mv)) return cudaErrorInvalidValue;
  cudaError_t e;
  BwdArgs args;
  args.tiles = tiles;
  args.ws = ws;
  args.offsets = offsets;
  args.lse = lse;
  args.dsum = dsum;
  args.dq_acc = dq_acc;
  args.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  args.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  args.b1 = bs.b1;
  args.db1 = bs.db1;
  args.T = p.total_tokens;
  args.h = p.h;
  args.m = p.m;
  args.scale = p.scale;
  args.scale_log2 = p.scale * 1.4426950408889634f;
  if constexpr (DH <= 64) {
    using H = BwdHalfCfg<DH>;
    auto hk = gdpa_bwd_half_kernel<DH, PHI, BIAS, kModeGdpa>;
    CUtensorMap mdq, mdv, mdk, unused_q, unused_g;
    if (!make_dq_map<DH>(p, dq_acc, &mdq)) return cudaErrorInvalidValue;
    // the outputs dV, dK have the layout (and so the maps) of the inputs K, V
    if (!make_bwd_maps<DH>(p, q, g, dk, dv, &unused_q, &unused_g, &mdk, &mdv))
      return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(hk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)H::SMEM);
    if (e != cudaSuccess) return e;
    KernelScope ks_("gdpa_bwd_sm100", st);
    hk<<<device_sm_count(), kHalfThreads, H::SMEM, st>>>(mq, mg, mk, mv, mdq, mdv, mdk, args);
    return cudaGetLastError();
  } else {
    using C = BwdCfg<DH>;
    auto kern = gdpa_bwd_sm100_kernel<DH, PHI, BIAS>;     // dh = 128 only
    CUtensorMap mdq;
    if (!make_dq_map<DH>(p, dq_acc, &mdq)) return cudaErrorInvalidValue;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    KernelScope ks_("gdpa_bwd_sm100", st);
    kern<<<device_sm_count(), kThreads, C::SMEM, st>>>(mq, mg, mk, mv, mdq, args);
    return cudaGetLastError();
  }
}

template <int DH, bool BIAS>
cudaError_t launch_bwd_dh(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                          const void* k, const void* v, const Bias& bs, const float* lse,
                          const float* dsum, const void* g, void* dk, void* dv, float* dq_acc,
                          WsHeader* ws, const Tile* tiles, cudaStream_t st) {
#define GDPA_BWD_PHI(PHIV) \
  launch_bwd_t<DH, PHIV, BIAS>(p, q, offsets, k, v, bs, lse, dsum, g, dk, dv, dq_acc, ws, tiles, st)
  switch (p.phi) {
    case GDPA_PHI_SOFTMAX: return GDPA_BWD_PHI(GDPA_PHI_SOFTMAX);
    case GDPA_PHI_SILU: return GDPA_BWD_PHI(GDPA_PHI_SILU);
    case GDPA_PHI_RELU: return GDPA_BWD_PHI(GDPA_PHI_RELU);
    case GDPA_PHI_GELU: return GDPA_BWD_PHI(GDPA_PHI_GELU);
    default: return GDPA_BWD_PHI(GDPA_PHI_IDENTITY);
  }
#undef GDPA_BWD_PHI
}

template <int DH>
cudaError_t launch_bwd_bias(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                            const void* k, const void* v, const Bias& bs, const float* lse,
                            const float* dsum, const void* g, void* dk, void* dv, float* dq_acc,
                            WsHeader* ws, const Tile* tiles, cudaStream_t st) {
  if (bs.b1 || bs.db1)
    return launch_bwd_dh<DH, true>(p, q, offsets, k, v, bs, lse, dsum, g, dk, dv, dq_acc, ws,
                                   tiles, st);
  return launch_bwd_dh<DH, false>(p, q, offsets, k, v, bs, lse, dsum, g, dk, dv, dq_acc, ws,
                                  tiles, st);
}

// Backward of seed pooling (POOL) or of the sliding window on the half
// kernel.  Maps: K, V, dK, dV are the jagged tokens [T, h, DH]; Q and dO are
// the tokens too (window) or the seeds [h, S, DH] and the pooled dO
// [B, h, S, DH] (pooling); the fp32 target of the dQ reduces is the token
// accumulator [T, h, DH] (window) or the seeds' gradient [h, S, DH] (pooling).
template <int DH, int MODE>
cudaError_t launch_jag_bwd_t(int B, int h, int S, int64_t T, int window, float scale,
                             const int32_t* offsets, const void* q, const void* g,
                             const void* k, const void* v, const float* lse, const float* dsum,
                             float* acc, void* dk, void* dv, WsHeader* ws, const Tile* tiles,
                             cudaStream_t st) {
  constexpr bool POOL = MODE == kModePool;
  constexpr int CH = DH < 64 ? DH : 64;
  using H = BwdHalfCfg<DH>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorInvalidValue;
  const CUtensorMapSwizzle sw = DH < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint32_t estr[3] = {1, 1, 1};
  auto map3 = [&](CUtensorMap* m, CUtensorMapDataType ty, int esz, const void* ptr,
                  cuuint64_t d1, cuuint64_t d2, cuuint32_t bx, cuuint32_t b1, cuuint32_t b2,
                  CUtensorMapSwizzle swz) -> bool {
    const cuuint64_t dims[3] = {(cuuint64_t)DH, d1, d2};
    const cuuint64_t str[2] = {(cuuint64_t)DH * esz, d1 * DH * esz};
    const cuuint32_t box[3] = {bx, b1, b2};
    return enc(m, ty, 3, const_cast<void*>(ptr), dims, str, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  const auto BF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const cuuint64_t Tm = T > 0 ? (cuuint64_t)T : 1;
  const CUtensorMapSwizzle swq = DH / 2 * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                                   : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap mq, mg, mk, mv, mdq, mdv, mdk;
  bool okm = map3(&mk, BF, 2, k, h, Tm, CH, 1, 128, sw) && map3(&mv, BF, 2, v, h, Tm, CH, 1, 128, sw) &&
             map3(&mdk, BF, 2, dk, h, Tm, CH, 1, 128, sw) &&
             map3(&mdv, BF, 2, dv, h, Tm, CH, 1, 128, sw);
  if (POOL)
    okm = okm && map3(&mq, BF, 2, q, S, h, CH, 128, 1, sw) &&
          map3(&mg, BF, 2, g, S, (cuuint64_t)B * h, CH, 128, 1, sw) &&
          map3(&mdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, acc, S, h, DH / 2, 32, 1, swq);
  else
    okm = okm && map3(&mq, BF, 2, q, h, Tm, CH, 1, 128, sw) &&
          map3(&mg, BF, 2, g, h, Tm, CH, 1, 128, sw) &&
          map3(&mdq, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, acc, h, Tm, DH / 2, 1, 32, swq);
  if (!okm) return cudaErrorInvalidValue;
  BwdArgs args = {};
  args.tiles = tiles;
  args.ws = ws;
  args.offsets = offsets;
  args.lse = lse;
  args.dsum = dsum;
  args.dq_acc = acc;
  args.dk = reinterpret_cast<__nv_bfloat16*>(dk);
  args.dv = reinterpret_cast<__nv_bfloat16*>(dv);
  args.T = T;
  args.h = h;
  args.m = 0;
  args.S = S;
  args.window = window;
  args.scale = scale;
  args.scale_log2 = scale * 1.4426950408889634f;
  auto hk = gdpa_bwd_half_kernel<DH, GDPA_PHI_SOFTMAX, false, MODE>;
  cudaError_t e = cudaFuncSetAttribute(hk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)H::SMEM);
  if (e != cudaSuccess) return e;
  KernelScope ks_(POOL ? "gdpa_pool_bwd_sm100" : "gdpa_window_bwd_sm100", st);
  hk<<<device_sm_count(), kHalfThreads, H::SMEM, st>>>(mq, mg, mk, mv, mdq, mdv, mdk, args);
  return cudaGetLastError();
}

template <int MODE>
cudaError_t launch_jag_bwd(int dh, int B, int h, int S, int64_t T, int window, float scale,
                           const int32_t* offsets, const void* q, const void* g, const void* k,
                           const void* v, const float* lse, const float* dsum, float* acc,
                           void* dk, void* dv, WsHeader* ws, const Tile* tiles, cudaStream_t st) {
  if (dh == 32)
    return launch_jag_bwd_t<32, MODE>(B, h, S, T, window, scale, offsets, q, g, k, v, lse, dsum,
                                      acc, dk, dv, ws, tiles, st);
  if (dh == 64)
    return launch_jag_bwd_t<64, MODE>(B, h, S, T, window, scale, offsets, q, g, k, v, lse, dsum,
                                      acc, dk, dv, ws, tiles, st);
  return cudaErrorInvalidValue;
}

template <int DH>
cudaError_t launch_prep(const void* o, const void* g, float* dsum, float* acc, int64_t acc_elems,
                        int64_t rows, int h, int64_t T, int flat, cudaStream_t st) {
  const int sms = device_sm_count();
  KernelScope ks_("gdpa_bwd_prep", st);
  bwd_prep_kernel<DH><<<sms * 8, 256, 0, st>>>(reinterpret_cast<const uint4*>(o),
                                               reinterpret_cast<const uint4*>(g), dsum,
                                               reinterpret_cast<float4*>(acc), acc_elems / 4,
                                               rows, h, T, 1, flat);
  return cudaGetLastError();
}

}  // namespace

// schedule (jagged key blocks) -> prep (zero the token dQ accumulator, D) ->
// half kernel in window mode -> dQ conversion.
cudaError_t launch_sm100_window_bwd(int B, int h, int dh, int64_t T, int max_n, int window,
                                    float scale, const int32_t* offsets, const void* q,
                                    const void* k, const void* v, const void* o,
                                    const float* lse, const void* dout, void* dq, void* dk,
                                    void* dv, float* dq_acc, float* dsum, WsHeader* ws,
                                    Tile* tiles, int64_t cap, cudaStream_t st) {
  cudaError_t e = launch_schedule_jkv(offsets, B, h, T, max_n, ws, tiles, cap, st);
  if (e != cudaSuccess || T == 0) return e;
  const int64_t rows = T * h;
  e = dh == 32 ? launch_prep<32>(o, dout, dsum, dq_acc, rows * dh, rows, h, T, 0, st)
               : launch_prep<64>(o, dout, dsum, dq_acc, rows * dh, rows, h, T, 0, st);
  if (e != cudaSuccess) return e;
  e = launch_jag_bwd<kModeWindow>(dh, B, h, 0, T, window, scale, offsets, q, dout, k, v, lse,
                                  dsum, dq_acc, dk, dv, ws, tiles, st);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  KernelScope ks_("gdpa_dq_convert", st);
  dq_convert_kernel<<<sms * 8, 256, 0, st>>>(reinterpret_cast<const float4*>(dq_acc),
                                              reinterpret_cast<uint4*>(dq), rows * dh / 8, scale);
  return cudaGetLastError();
}

// schedule (jagged key blocks) -> prep (zero dseeds, D of the pooled rows) ->
// half kernel in pooling mode (dseeds accumulates over every sample) -> scale.
cudaError_t launch_sm100_pool_bwd(int B, int h, int dh, int S, int64_t T, int max_n, float scale,
                                  const int32_t* offsets, const void* seeds, const void* k,
                                  const void* v, const void* o, const float* lse,
                                  const void* dout, float* dseeds, void* dk, void* dv,
                                  float* dsum, WsHeader* ws, Tile* tiles, int64_t cap,
                                  cudaStream_t st) {
  cudaError_t e = launch_schedule_jkv(offsets, B, h, T, max_n, ws, tiles, cap, st);
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)B * h * S, nseed = (int64_t)h * S * dh;
  e = dh == 32 ? launch_prep<32>(o, dout, dsum, dseeds, nseed, rows, h, T, 1, st)
               : launch_prep<64>(o, dout, dsum, dseeds, nseed, rows, h, T, 1, st);
  if (e != cudaSuccess) return e;
  if (T > 0) {
    e = launch_jag_bwd<kModePool>(dh, B, h, S, T, 0, scale, offsets, seeds, dout, k, v, lse, dsum,
                                  dseeds, dk, dv, ws, tiles, st);
    if (e != cudaSuccess) return e;
  }
  const int sms = device_sm_count();
  KernelScope ks_("gdpa_seed_scale", st);
  scale_f32_kernel<<<sms * 4, 256, 0, st>>>(dseeds, nseed, scale);
  return cudaGetLastError();
}

int64_t sm100_bwd_items(const gdpa_problem_t& p) {
  return (int64_t)p.B * p.h * ((p.m + 127) / 128);
}

// schedule (LPT list) -> prep (zero dQ accumulator, softmax D) -> [bias terms]
// -> fused backward -> dQ conversion.
cudaError_t launch_sm100_bwd(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                             const void* k, const void* v, const Bias& bs, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             float* dq_acc, float* dsum, WsHeader* ws, Tile* tiles,
                             cudaStream_t st) {
  cudaError_t e = launch_schedule_kv(p, offsets, ws, tiles, st);
  if (e != cudaSuccess) return e;
  const int64_t rows = p.total_tokens * p.h;
  const int sms = device_sm_count();
  const bool softmax = p.phi == GDPA_PHI_SOFTMAX;
  if (rows > 0) {
    KernelScope ks_("gdpa_bwd_prep", st);
    auto prep = p.dh == 32 ? bwd_prep_kernel<32> : p.dh == 64 ? bwd_prep_kernel<64>
                                                              : bwd_prep_kernel<128>;
    // with an output bias the softmax row sums come from the bias kernel (O - b2)
    prep<<<sms * 8, 256, 0, st>>>(reinterpret_cast<const uint4*>(o),
                                  reinterpret_cast<const uint4*>(dout), dsum,
                                  reinterpret_cast<float4*>(dq_acc), rows * p.dh / 4, rows, p.h,
                                  p.total_tokens, softmax && !bs.b2 ? 1 : 0, 0);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  e = launch_bias_prep(p, offsets, o, dout, bs.b2, softmax && bs.b2 ? dsum : nullptr, bs.db1,
                       bs.db2, ws, st);
  if (e != cudaSuccess) return e;
  switch (p.dh) {
    case 32: e = launch_bwd_bias<32>(p, q, offsets, k, v, bs, lse, dsum, dout, dk, dv, dq_acc, ws, tiles, st); break;
    case 64: e = launch_bwd_bias<64>(p, q, offsets, k, v, bs, lse, dsum, dout, dk, dv, dq_acc, ws, tiles, st); break;
    case 128: e = launch_bwd_bias<128>(p, q, offsets, k, v, bs, lse, dsum, dout, dk, dv, dq_acc, ws, tiles, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || rows == 0) return e;
  KernelScope ks_("gdpa_dq_convert", st);
  dq_convert_kernel<<<sms * 8, 256, 0, st>>>(reinterpret_cast<const float4*>(dq_acc),
                                              reinterpret_cast<uint4*>(dq), rows * p.dh / 8,
                                              p.scale);
  return cudaGetLastError();
}

}  // namespace gdpa
