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
// dQ_i (lane = query row) is added into an fp32 workspace with vector
// reductions; a last kernel scales it by s and rounds it to bf16.
//
// CTA = 12 warps, one persistent CTA per SM, static round-robin over a work
// list sorted by sample length (longest first):
//   warp 0 TMA producer, warp 1 MMA issuer, warp 2 TMEM allocator,
//   warps 4-7 and 8-11: the two activation groups, splitting each query tile's
//   128 rows in halves; they also drain dQ_i and, at the end of an item, store
//   dV (group 0) and dK (group 1).
#include <cudaTypedefs.h>
#include <math.h>

#include "gdpa_internal.cuh"
#include "sm100.cuh"

namespace gdpa {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
int device_sm_count();

namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// ---------------------------------------------------------------- prep / convert

// Zeroes the fp32 dQ workspace and, for softmax, writes D[head, t] =
// sum_d dO[t, head, d] * O[t, head, d] (one warp per (t, head) row).
__global__ void bwd_prep_kernel(const __nv_bfloat16* __restrict__ o,
                                const __nv_bfloat16* __restrict__ g, float* __restrict__ dsum,
                                float4* __restrict__ dq_acc, int64_t rows, int h, int dh,
                                int64_t T, int softmax) {
  const int64_t n4 = rows * dh / 4;
  const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t nth = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = tid; i < n4; i += nth) dq_acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  if (!softmax) return;
  const int lane = threadIdx.x & 31;
  for (int64_t row = tid >> 5; row < rows; row += nth >> 5) {
    float acc = 0.f;
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(o + row * dh);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(g + row * dh);
    for (int d = lane; d < dh / 2; d += 32) {
      const float2 a = __bfloat1622float2(o2[d]), b = __bfloat1622float2(g2[d]);
      acc = fmaf(a.x, b.x, fmaf(a.y, b.y, acc));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) dsum[(int64_t)(row % h) * T + row / h] = acc;
  }
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
  int64_t T;
  int h, m;
  float scale, scale_log2;
};

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
  static constexpr uint32_t COL_DQ = DH <= 64 ? 256 + 2 * DH : COL_DP;
  // barriers
  static constexpr int B_KVFULL = 0, B_KVEMPTY = 1, B_SFULL = 2, B_PFULL = 3, B_DQFULL = 4,
                       B_DQEMPTY = 5, B_ACCFULL = 6, B_ACCEMPTY = 7, B_DRAIN = 8,
                       B_STFULL = 9, B_STEMPTY = 9 + NSTG, NBAR = 9 + 2 * NSTG;
  static constexpr uint32_t OFF_K = 0, OFF_V = TILEB, OFF_STG = 2 * TILEB;
  static constexpr uint32_t OFF_DS = OFF_STG + NSTG * 2 * TILEB;
  static constexpr uint32_t OFF_CTL = OFF_DS + DSB;
  static constexpr uint32_t CTL_BYTES = 1024 + 8 * 2 * 128 * 4;  // barriers + per-warp row stats
  static constexpr uint32_t SMEM_USED = 1024 + OFF_CTL + CTL_BYTES;
  static constexpr uint32_t SMEM = SMEM_USED > 120u * 1024u ? SMEM_USED : 120u * 1024u;
};
