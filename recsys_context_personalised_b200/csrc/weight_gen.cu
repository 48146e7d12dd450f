// Weight Generation for sm_100a: each sample's GDPA keys (or values) from its
// context vector, on the tcgen05 tensor cores.
//
// The Kunlun summary (section 2.1) lists Weight Generation in the Interaction
// Block, and the RecSysChannel review ("Kunlun ... [2/2]", item 1) says that
// K and V are obtained from the context features; the pages give no formula.
// The reading taken is a learned linear map per output tensor:
//   y[b, f] = sum_c w[f, c] * ctx[b, c],   f < F = h * m * dh,
// with y[b] viewed as [h, m, dh] (K_b or V_b) and rounded to bf16.
//
// As a GEMM: D[b, f] = ctx[b, :] . w[f, :], M = samples, N = features,
// K = C (the context length, 32 or 64).  w and ctx are fp32 and enter the
// tensor core as tf32 (kind::tf32, fp32 accumulation): tf32 keeps 10 mantissa
// bits, well inside the bf16 rounding of the output.  The output is HBM-bound
// (2 bytes written per 2 C flops), so the kernel is built around the stores.
//
// One persistent CTA per SM; work item = a 128-feature tile of w, loaded once
// and kept in shared memory while the CTA loops over all 128-sample tiles of
// ctx (ctx is small and stays in L2).  Warp 0: TMA producer (w tile, a
// two-slot ctx ring); warp 1: MMA issuer (D in TMEM, two 128-column
// accumulators); warp 2: TMEM allocator; warps 4-7: epilogue (TMEM -> bf16 ->
// 128B-swizzled staging box -> bulk tensor store, which clips rows >= B and
// columns >= F).
#include <cudaTypedefs.h>

#include "gdpa_internal.cuh"
#include "sm100.cuh"

namespace gdpa {

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
int device_sm_count();

namespace {

using namespace sm100;

constexpr int kWgThreads = 256;
constexpr uint64_t kWgTimeoutNs = 2000000000ull;

template <int C>
struct WgCfg {
  static constexpr int BM = 128, BN = 128;              // samples x features per tile
  static constexpr int NCH = C / 32;                    // 32-fp32 (128 B) chunks along C
  static constexpr uint32_t CHUNKB = 128 * 128;         // [128 rows x 32 fp32]
  static constexpr uint32_t TILEB = NCH * CHUNKB;       // [128 rows x C] fp32
  static constexpr uint32_t OFF_W = 0;                  // two w slots
  static constexpr uint32_t OFF_X = 2 * TILEB;          // two ctx slots
  static constexpr uint32_t OFF_Y = 4 * TILEB;          // [128 x 128] bf16 staging: 2 boxes of 64 columns
  static constexpr uint32_t YBOXB = 128 * 128;          // [128 rows x 64 bf16]
  static constexpr uint32_t OFF_CTL = OFF_Y + 2 * YBOXB;
  static constexpr int B_WFULL = 0, B_WEMPTY = 2, B_XFULL = 4, B_XEMPTY = 6, B_AFULL = 8,
                       B_AEMPTY = 10, B_DRAIN = 12, NBAR = 13;
  static constexpr uint32_t SMEM = 1024 + OFF_CTL + 1024;
  static_assert(SMEM <= 232448u, "exceeds the 227 KB of shared memory a CTA can have");
  static_assert(8 * NBAR + 8 <= 1024, "control block");
};

// tf32 x tf32 -> fp32 instruction descriptor (A, B K-major): formats 2 = TF32.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(m), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(m),
      "r"(src), "r"(c0), "r"(c1)
      : "memory");
}

struct WgArgs {
  int nB, nF;            // 128-sample and 128-feature tiles
  WsHeader* status;      // GDPA_ERR_TIMEOUT on a bounded-wait expiry (may be NULL)
};

template <int C>
__global__ void __launch_bounds__(kWgThreads, 1)
weight_gen_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ CUtensorMap tmY, const WgArgs a) {
  using G = WgCfg<C>;
  constexpr uint32_t IDESC = idesc_tf32(G::BM, G::BN);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* ctl = smem_raw + (base - raw) + G::OFF_CTL;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * G::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * G::NBAR + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(G::B_WFULL + i), 1);
      mbar_init(bar(G::B_WEMPTY + i), 1);
      mbar_init(bar(G::B_XFULL + i), 1);
      mbar_init(bar(G::B_XEMPTY + i), 1);
      mbar_init(bar(G::B_AFULL + i), 1);
      mbar_init(bar(G::B_AEMPTY + i), 128);
    }
    mbar_init(bar(G::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmY);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    uint32_t ic = 0, xc = 0;
    bool ok = true;
    for (int ft = blockIdx.x; ok && ft < a.nF; ft += gridDim.x, ++ic) {
      const uint32_t ws = ic & 1u;
      if (!mbar_wait(bar(G::B_WEMPTY + ws), ((ic >> 1) & 1u) ^ 1u, abort_flag, kWgTimeoutNs)) break;
      mbar_expect_tx(bar(G::B_WFULL + ws), G::TILEB);
      for (int c = 0; c < G::NCH; ++c)
        tma_load_2d(base + G::OFF_W + ws * G::TILEB + c * G::CHUNKB, &tmW, bar(G::B_WFULL + ws),
                    32 * c, ft * G::BN);
      for (int bt = 0; bt < a.nB; ++bt, ++xc) {
        const uint32_t xs = xc & 1u;
        if (!mbar_wait(bar(G::B_XEMPTY + xs), ((xc >> 1) & 1u) ^ 1u, abort_flag, kWgTimeoutNs)) {
          ok = false;
          break;
        }
        mbar_expect_tx(bar(G::B_XFULL + xs), G::TILEB);
        for (int c = 0; c < G::NCH; ++c)
          tma_load_2d(base + G::OFF_X + xs * G::TILEB + c * G::CHUNKB, &tmX, bar(G::B_XFULL + xs),
                      32 * c, bt * G::BM);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t ic = 0, xc = 0, tc = 0;
    bool ok = true;
    for (int ft = blockIdx.x; ok && ft < a.nF; ft += gridDim.x, ++ic) {
      const uint32_t ws = ic & 1u;
      if (!mbar_wait(bar(G::B_WFULL + ws), (ic >> 1) & 1u, abort_flag, kWgTimeoutNs)) break;
      tc_fence_after();
      const uint64_t b0 = smem_desc(base + G::OFF_W + ws * G::TILEB, 16, 1024, kSw128);
      for (int bt = 0; bt < a.nB; ++bt, ++xc, ++tc) {
        const uint32_t xs = xc & 1u, as = tc & 1u;
        if (!mbar_wait(bar(G::B_XFULL + xs), (xc >> 1) & 1u, abort_flag, kWgTimeoutNs) ||
            !mbar_wait(bar(G::B_AEMPTY + as), ((tc >> 1) & 1u) ^ 1u, abort_flag, kWgTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t a0 = smem_desc(base + G::OFF_X + xs * G::TILEB, 16, 1024, kSw128);
#pragma unroll
        for (int k = 0; k < C / 8; ++k) {               // 8 tf32 (32 B) per instruction
          const uint32_t off = (k / 4) * G::CHUNKB + (k % 4) * 32;
          mma_tf32(tmem + as * G::BN, desc_advance(a0, off), desc_advance(b0, off), IDESC,
                   k > 0 ? 1u : 0u);
        }
        mma_commit(bar(G::B_XEMPTY + xs));
        mma_commit(bar(G::B_AFULL + as));
      }
      mma_commit(bar(G::B_WEMPTY + ws));
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;                    // sample row within the tile
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t tc = 0;
    bool ok = true;
    for (int ft = blockIdx.x; ok && ft < a.nF; ft += gridDim.x) {
      for (int bt = 0; bt < a.nB; ++bt, ++tc) {
        const uint32_t as = tc & 1u;
        const bool w = mbar_wait(bar(G::B_AFULL + as), (tc >> 1) & 1u, abort_flag, kWgTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld_x32(tmem + lane_off + as * G::BN + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(G::B_AEMPTY + as));            // the accumulator is free
        // the previous tile's bulk stores must have read the staging boxes
        if (threadIdx.x == 128) bulk_wait_group_read0();
        named_bar_sync(1, 128);
#pragma unroll
        for (int bx = 0; bx < 2; ++bx) {
          const uint32_t box = base + G::OFF_Y + bx * G::YBOXB + (uint32_t)row * 128;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t* s = &v[64 * bx + 8 * j];
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                         ::"r"(box + (((uint32_t)j ^ (uint32_t)(row & 7)) << 4)),
                         "r"(pack_bf16x2(__uint_as_float(s[0]), __uint_as_float(s[1]))),
                         "r"(pack_bf16x2(__uint_as_float(s[2]), __uint_as_float(s[3]))),
                         "r"(pack_bf16x2(__uint_as_float(s[4]), __uint_as_float(s[5]))),
                         "r"(pack_bf16x2(__uint_as_float(s[6]), __uint_as_float(s[7])))
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (threadIdx.x == 128) {
          tma_store_2d(&tmY, base + G::OFF_Y, ft * G::BN, bt * G::BM);
          tma_store_2d(&tmY, base + G::OFF_Y + G::YBOXB, ft * G::BN + 64, bt * G::BM);
          bulk_commit_group();
        }
      }
    }
    if (threadIdx.x == 128) bulk_wait_group0();         // stores complete before exit
  }

  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    if (a.status) report(a.status, GDPA_ERR_TIMEOUT);
    volatile int never = 0;
    if (warp == 1 && lane == 0) {
      mma_commit(bar(G::B_DRAIN));
      mbar_wait(bar(G::B_DRAIN), 0, &never, kWgTimeoutNs);
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
  if (warp == 2) tmem_dealloc(tmem, 256);
}

bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, void* ptr, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, dt, 2, ptr, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int C>
cudaError_t launch_wg(int B, int64_t F, const float* w, const float* ctx, void* y,
                      WsHeader* status, cudaStream_t st) {
  using G = WgCfg<C>;
  CUtensorMap mw, mx, my;
  if (!encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float*>(w), C, (uint64_t)F,
                 (uint64_t)C * 4, 32, 128) ||
      !encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, const_cast<float*>(ctx), C, (uint64_t)B,
                 (uint64_t)C * 4, 32, 128) ||
      !encode_2d(&my, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, (uint64_t)F, (uint64_t)B,
                 (uint64_t)F * 2, 64, 128))
    return cudaErrorInvalidValue;
  auto kern = weight_gen_kernel<C>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)G::SMEM);
  if (e != cudaSuccess) return e;
  WgArgs args;
  args.nB = (B + G::BM - 1) / G::BM;
  args.nF = (int)((F + G::BN - 1) / G::BN);
  args.status = status;
  const int grid = args.nF < device_sm_count() ? args.nF : device_sm_count();
  KernelScope ks_("gdpa_weight_gen", st);
  kern<<<grid, kWgThreads, G::SMEM, st>>>(mw, mx, my, args);
  return cudaGetLastError();
}

}  // namespace
}  // namespace gdpa

using namespace gdpa;

extern "C" gdpa_status_t gdpa_weight_gen(int32_t B, int64_t F, int32_t C, const float* w,
                                         const float* ctx, void* y, void* status_ws,
                                         void* stream) {
  if (B < 0 || F < 0 || (C != 32 && C != 64)) return GDPA_ERR_UNSUPPORTED;
  if (F % 8 != 0 || F / 128 >= ((int64_t)1 << 31)) return GDPA_ERR_UNSUPPORTED;
  if (B == 0 || F == 0) return GDPA_OK;
  if (!w || !ctx || !y || ((uintptr_t)w & 15u) || ((uintptr_t)ctx & 15u) || ((uintptr_t)y & 15u))
    return GDPA_ERR_INVALID_ARG;
  if (status_ws && ((uintptr_t)status_ws & 255u)) return GDPA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* status = (WsHeader*)status_ws;
  if (status && cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess)
    return GDPA_ERR_CUDA;
  cudaError_t e;
  if (C == 32)
    e = launch_wg<32>(B, F, w, ctx, y, status, st);
  else
    e = launch_wg<64>(B, F, w, ctx, y, status, st);
  return e == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Backward of the Weight Generation map for an upstream dy [B, F] (bf16):
//   dw[f, c]   = sum_b dy[b, f] * ctx[b, c]      (fp32 [F, C])
//   dctx[b, c] = sum_f dy[b, f] * w[f, c]        (fp32 [B, C])
// Both contractions read each dy tile once, from the same shared-memory
// bytes: dw as dy^T ctx (A = the dy tile read MN-major, B = ctx read
// MN-major) and dctx as dy w (A = the dy tile read K-major, B = w read
// MN-major), on kind::f16 tensor cores with bf16 operands: a prep kernel
// rounds ctx and w to bf16 into the workspace and clears dctx.
//
// Work item = a 128-feature tile: the CTA loops over all 128-sample tiles,
// accumulating the dw tile in TMEM (64 columns) and its share of dctx in one
// 64-column TMEM accumulator per sample tile (so B <= 7 * 128); the dw tile
// leaves through a staging box and bulk tensor stores, and at the end each
// CTA adds its dctx share into the fp32 output with vector reductions.
namespace gdpa {
namespace {

constexpr int kWgbMaxSampleTiles = 7;

struct WgbCfg {
  static constexpr int C = 64;
  static constexpr uint32_t WTILE = 128 * 128;          // [128 f x 64 c] bf16
  static constexpr uint32_t DYTILE = 2 * 128 * 128;     // [128 b x 128 f] bf16, two 64-f boxes
  static constexpr uint32_t XTILE = 128 * 128;          // [128 b x 64 c] bf16
  static constexpr uint32_t STAGE = DYTILE + XTILE;
  static constexpr uint32_t OFF_W = 0;                  // two w slots
  static constexpr uint32_t OFF_ST = 2 * WTILE;         // two (dy, ctx) stages
  static constexpr uint32_t OFF_DW = OFF_ST + 2 * STAGE;   // dw staging: two [128 x 32 fp32] boxes
  static constexpr uint32_t OFF_CTL = OFF_DW + 2 * 128 * 128;
  static constexpr int B_WFULL = 0, B_WEMPTY = 2, B_SFULL = 4, B_SEMPTY = 6, B_DWFULL = 8,
                       B_DWEMPTY = 9, B_XFULL = 10, B_DRAIN = 11, NBAR = 12;
  static constexpr uint32_t SMEM = 1024 + OFF_CTL + 1024;
  static_assert(SMEM <= 232448u, "exceeds the 227 KB of shared memory a CTA can have");
};

__global__ void wg_bwd_prep_kernel(const float4* __restrict__ w, const float4* __restrict__ ctx,
                                   uint2* __restrict__ w16, uint2* __restrict__ ctx16,
                                   float4* __restrict__ dctx, int64_t nw4, int64_t nc4) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nw4 + nc4; i += stride) {
    const float4 x = i < nw4 ? w[i] : ctx[i - nw4];
    const uint2 p = make_uint2(pack_bf16x2(x.x, x.y), pack_bf16x2(x.z, x.w));
    if (i < nw4) {
      w16[i] = p;
    } else {
      ctx16[i - nw4] = p;
      dctx[i - nw4] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

struct WgbArgs {
  int B, nB, nF;
  int64_t F;
  float* dctx;
  WsHeader* status;
};

__global__ void __launch_bounds__(kWgThreads, 1)
weight_gen_bwd_kernel(const __grid_constant__ CUtensorMap tmDY,
                      const __grid_constant__ CUtensorMap tmX16,
                      const __grid_constant__ CUtensorMap tmW16,
                      const __grid_constant__ CUtensorMap tmDW, const WgbArgs a) {
  using G = WgbCfg;
  constexpr uint32_t IDESC_DW = idesc_bf16(128, 64, 1, 1);     // dy^T (MN-major) x ctx (MN-major)
  constexpr uint32_t IDESC_DX = idesc_bf16(128, 64, 0, 1);     // dy (K-major) x w (MN-major)
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* ctl = smem_raw + (base - raw) + G::OFF_CTL;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * G::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * G::NBAR + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // TMEM: dw accumulator [0, 64), dctx of sample tile t at [64 + 64 t, 128 + 64 t)
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(G::B_WFULL + i), 1);
      mbar_init(bar(G::B_WEMPTY + i), 1);
      mbar_init(bar(G::B_SFULL + i), 1);
      mbar_init(bar(G::B_SEMPTY + i), 1);
    }
    mbar_init(bar(G::B_DWFULL), 1);
    mbar_init(bar(G::B_DWEMPTY), 128);
    mbar_init(bar(G::B_XFULL), 1);
    mbar_init(bar(G::B_DRAIN), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmDY);
    prefetch_tmap(&tmX16);
    prefetch_tmap(&tmW16);
    prefetch_tmap(&tmDW);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    uint32_t ic = 0, sc = 0;
    bool ok = true;
    for (int ft = blockIdx.x; ok && ft < a.nF; ft += gridDim.x, ++ic) {
      const uint32_t ws = ic & 1u;
      if (!mbar_wait(bar(G::B_WEMPTY + ws), ((ic >> 1) & 1u) ^ 1u, abort_flag, kWgTimeoutNs)) break;
      mbar_expect_tx(bar(G::B_WFULL + ws), G::WTILE);
      tma_load_2d(base + G::OFF_W + ws * G::WTILE, &tmW16, bar(G::B_WFULL + ws), 0, ft * 128);
      for (int bt = 0; bt < a.nB; ++bt, ++sc) {
        const uint32_t ss = sc & 1u;
        if (!mbar_wait(bar(G::B_SEMPTY + ss), ((sc >> 1) & 1u) ^ 1u, abort_flag, kWgTimeoutNs)) {
          ok = false;
          break;
        }
        const uint32_t st = base + G::OFF_ST + ss * G::STAGE;
        mbar_expect_tx(bar(G::B_SFULL + ss), G::STAGE);
        tma_load_2d(st, &tmDY, bar(G::B_SFULL + ss), ft * 128, bt * 128);
        tma_load_2d(st + G::DYTILE / 2, &tmDY, bar(G::B_SFULL + ss), ft * 128 + 64, bt * 128);
        tma_load_2d(st + G::DYTILE, &tmX16, bar(G::B_SFULL + ss), 0, bt * 128);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t ic = 0, sc = 0;
    bool ok = true;
    for (int ft = blockIdx.x; ok && ft < a.nF; ft += gridDim.x, ++ic) {
      const uint32_t ws = ic & 1u;
      if (!mbar_wait(bar(G::B_WFULL + ws), (ic >> 1) & 1u, abort_flag, kWgTimeoutNs) ||
          !mbar_wait(bar(G::B_DWEMPTY), (ic & 1u) ^ 1u, abort_flag, kWgTimeoutNs))
        break;
      tc_fence_after();
      const uint64_t wdesc = smem_desc(base + G::OFF_W + ws * G::WTILE, 16, 1024, kSw128);
      for (int bt = 0; bt < a.nB; ++bt, ++sc) {
        const uint32_t ss = sc & 1u;
        if (!mbar_wait(bar(G::B_SFULL + ss), (sc >> 1) & 1u, abort_flag, kWgTimeoutNs)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = base + G::OFF_ST + ss * G::STAGE;
        // dw[f, c] += sum_b dy[b, f] ctx[b, c]: K = the tile's 128 samples, 16 per step
        const uint64_t dyT = smem_desc(st, G::DYTILE / 2, 1024, kSw128);   // MN-major, 64-f atoms
        const uint64_t xmn = smem_desc(st + G::DYTILE, 16, 1024, kSw128);  // MN-major, one 64-c atom
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem, desc_advance(dyT, k * 2048), desc_advance(xmn, k * 2048), IDESC_DW,
                 (bt > 0 || k > 0) ? 1u : 0u);
        // dctx[b, c] += sum_f dy[b, f] w[f, c]: K = the tile's 128 features, 16 per step
        const uint64_t dyK = smem_desc(st, 16, 1024, kSw128);               // K-major, two 64-f chunks
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t off = (k / 4) * (G::DYTILE / 2) + (k % 4) * 32;
          mma_ss(tmem + 64 + 64 * bt, desc_advance(dyK, off), desc_advance(wdesc, k * 2048),
                 IDESC_DX, (ic > 0 || k > 0) ? 1u : 0u);
        }
        mma_commit(bar(G::B_SEMPTY + ss));
      }
      mma_commit(bar(G::B_WEMPTY + ws));
      mma_commit(bar(G::B_DWFULL));
    }
    mma_commit(bar(G::B_XFULL));                        // every dctx product has completed
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    uint32_t ic = 0;
    bool ok = true;
    for (int ft = blockIdx.x; ok && ft < a.nF; ft += gridDim.x, ++ic) {
      const bool w = mbar_wait(bar(G::B_DWFULL), ic & 1u, abort_flag, kWgTimeoutNs);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t v[64];
      tmem_ld_x32(tmem + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld_x32(tmem + lane_off + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(G::B_DWEMPTY));
      if (threadIdx.x == 128) bulk_wait_group_read0();
      named_bar_sync(1, 128);
      // dw row `row` of the tile: two [128 x 32 fp32] boxes, 128B swizzle
#pragma unroll
      for (int bx = 0; bx < 2; ++bx) {
        const uint32_t box = base + G::OFF_DW + bx * 128 * 128 + (uint32_t)row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                       ::"r"(box + (((uint32_t)j ^ (uint32_t)(row & 7)) << 4)),
                       "r"(v[32 * bx + 4 * j]), "r"(v[32 * bx + 4 * j + 1]),
                       "r"(v[32 * bx + 4 * j + 2]), "r"(v[32 * bx + 4 * j + 3])
                       : "memory");
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (threadIdx.x == 128) {
        tma_store_2d(&tmDW, base + G::OFF_DW, 0, ft * 128);
        tma_store_2d(&tmDW, base + G::OFF_DW + 128 * 128, 32, ft * 128);
        bulk_commit_group();
      }
    }
    // this CTA's share of dctx: one reduction per 4 values of each sample row
    if (ok && blockIdx.x < a.nF) {
      const bool w = mbar_wait(bar(G::B_XFULL), 0, abort_flag, kWgTimeoutNs);
      if (__all_sync(0xffffffffu, w)) {
        tc_fence_after();
        for (int bt = 0; bt < a.nB; ++bt) {
          uint32_t v[64];
          tmem_ld_x32(tmem + lane_off + 64 + 64 * bt, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
          tmem_ld_x32(tmem + lane_off + 96 + 64 * bt, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
          tmem_wait_ld();
          const int b = bt * 128 + row;
          if (b < a.B) {
            float* dst = a.dctx + (int64_t)b * G::C;
#pragma unroll
            for (int j = 0; j < 16; ++j)
              red_add_v4(dst + 4 * j, __uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                         __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          }
        }
      }
    }
    if (threadIdx.x == 128) bulk_wait_group0();
  }

  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    if (a.status) report(a.status, GDPA_ERR_TIMEOUT);
    volatile int never = 0;
    if (warp == 1 && lane == 0) {
      mma_commit(bar(G::B_DRAIN));
      mbar_wait(bar(G::B_DRAIN), 0, &never, kWgTimeoutNs);
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

struct WgbLayout {
  size_t w16_off, x16_off, total;
};

WgbLayout wgb_layout(int B, int64_t F) {
  WgbLayout L;
  L.w16_off = sizeof(WsHeader);
  L.x16_off = align_up(L.w16_off + (size_t)F * WgbCfg::C * 2, 256);
  L.total = align_up(L.x16_off + (size_t)B * WgbCfg::C * 2, 256);
  return L;
}

gdpa_status_t wgb_check(int32_t B, int64_t F, int32_t C) {
  if (B < 0 || F < 0) return GDPA_ERR_INVALID_ARG;
  if (C != WgbCfg::C || F % 8 != 0 || B > kWgbMaxSampleTiles * 128 ||
      F / 128 >= ((int64_t)1 << 31))
    return GDPA_ERR_UNSUPPORTED;
  return GDPA_OK;
}

}  // namespace
}  // namespace gdpa

extern "C" gdpa_status_t gdpa_weight_gen_bwd_workspace_size(int32_t B, int64_t F, int32_t C,
                                                             size_t* bytes) {
  const gdpa_status_t s = wgb_check(B, F, C);
  if (s != GDPA_OK) return s;
  if (!bytes) return GDPA_ERR_INVALID_ARG;
  *bytes = wgb_layout(B, F).total;
  return GDPA_OK;
}

extern "C" gdpa_status_t gdpa_weight_gen_bwd(int32_t B, int64_t F, int32_t C, const float* w,
                                             const float* ctx, const void* dy, float* dw,
                                             float* dctx, void* workspace, size_t workspace_bytes,
                                             void* stream) {
  gdpa_status_t s = wgb_check(B, F, C);
  if (s != GDPA_OK) return s;
  if (B == 0 || F == 0) return GDPA_OK;
  if (!w || !ctx || !dy || !dw || !dctx || ((uintptr_t)w & 15u) || ((uintptr_t)ctx & 15u) ||
      ((uintptr_t)dy & 15u) || ((uintptr_t)dw & 15u) || ((uintptr_t)dctx & 15u))
    return GDPA_ERR_INVALID_ARG;
  const WgbLayout L = wgb_layout(B, F);
  if (!workspace || ((uintptr_t)workspace & 255u) || workspace_bytes < L.total)
    return GDPA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* status = (WsHeader*)workspace;
  __nv_bfloat16* w16 = (__nv_bfloat16*)((char*)workspace + L.w16_off);
  __nv_bfloat16* x16 = (__nv_bfloat16*)((char*)workspace + L.x16_off);
  if (cudaMemsetAsync(status, 0, sizeof(int32_t), st) != cudaSuccess) return GDPA_ERR_CUDA;
  const int sms = device_sm_count();
  {
    KernelScope ks_("gdpa_weight_gen_bwd_prep", st);
    wg_bwd_prep_kernel<<<sms * 4, 256, 0, st>>>(
        reinterpret_cast<const float4*>(w), reinterpret_cast<const float4*>(ctx),
        reinterpret_cast<uint2*>(w16), reinterpret_cast<uint2*>(x16),
        reinterpret_cast<float4*>(dctx), F * WgbCfg::C / 4, (int64_t)B * WgbCfg::C / 4);
    if (cudaGetLastError() != cudaSuccess) return GDPA_ERR_CUDA;
  }
  CUtensorMap mdy, mx, mw, mdw;
  if (!encode_2d(&mdy, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, const_cast<void*>(dy), (uint64_t)F,
                 (uint64_t)B, (uint64_t)F * 2, 64, 128) ||
      !encode_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x16, 64, (uint64_t)B, 128, 64, 128) ||
      !encode_2d(&mw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w16, 64, (uint64_t)F, 128, 64, 128) ||
      !encode_2d(&mdw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, dw, 64, (uint64_t)F, 256, 32, 128))
    return GDPA_ERR_CUDA;
  auto kern = weight_gen_bwd_kernel;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)WgbCfg::SMEM) != cudaSuccess)
    return GDPA_ERR_CUDA;
  WgbArgs args;
  args.B = B;
  args.nB = (B + 127) / 128;
  args.nF = (int)((F + 127) / 128);
  args.F = F;
  args.dctx = dctx;
  args.status = status;
  const int grid = args.nF < sms ? args.nF : sms;
  KernelScope ks_("gdpa_weight_gen_bwd", st);
  kern<<<grid, kWgThreads, WgbCfg::SMEM, st>>>(mdy, mx, mw, mdw, args);
  return cudaGetLastError() == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}
