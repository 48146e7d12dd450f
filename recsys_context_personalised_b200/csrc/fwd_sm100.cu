// Fused GDPA forward for sm_100a: TMA + tcgen05 (TMEM accumulators).
//
// Operator (Kunlun summary, section 2.2, GDPA bullet: PFFN recast as a
// multi-head attention operator fused into one FlashAttention-like kernel;
// RecSysChannel review "Kunlun ... [2/2]", items 1-2: K and V come from the
// context features, the event sequence is turned into Q).  Per query tile
// (sample b, head j, up to 128 rows) and per 128-key block:
//   S = Q K^T            tcgen05.mma, A and B from shared memory, S in TMEM
//   P = phi(s S)         activation warps: TMEM -> registers -> TMEM (bf16)
//   O += P V             tcgen05.mma, A = P from TMEM, B = V from shared memory
// softmax keeps running row statistics (online softmax, rescaling O only when
// the running max grows by more than 2^8); the elementwise phi needs none.
//
// Each work item is a pair of consecutive tiles of the jagged tile list, A and
// B, processed side by side: the MMA issuer interleaves their two dependency
// chains (S_A, S_B, PV_A, S_A', PV_B, S_B', ...) so the tensor core always has
// the other tile's work queued while one tile's activation runs.  When A and B
// belong to the same (sample, head) they share every K/V block load; otherwise
// each streams its own.
//
// CTA = 12 warps, one persistent CTA per SM, static round-robin over the pairs:
//   warp 0      TMA producer (one lane)
//   warp 1      MMA issuer (one lane)
//   warp 2      TMEM allocator
//   warps 4-7   activation group A (tile A), warps 8-11 group B (tile B)
//
// TMEM columns (512 allocated): S_A [0,128), S_B [128,256) (P_X aliases the
// first 64 columns of S_X as packed bf16), O_A [256, 256+dh), O_B [256+dh, 256+2dh).
#include <cudaTypedefs.h>
#include <math.h>

#include "gdpa_internal.cuh"
#include "sm100.cuh"

namespace gdpa {

// cuTensorMapEncodeTiled through the runtime's driver entry-point query (no
// link-time dependency on libcuda).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

int device_sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

namespace {

using namespace sm100;

constexpr int kThreads = 384;
constexpr uint64_t kTimeoutNs = 2000000000ull;   // 2 s per wait; a healthy wait is microseconds

struct FwdArgs {
  const Tile* tiles;
  WsHeader* ws;
  __nv_bfloat16* o;
  float* lse;
  const float* b1;   // [B, h, m] key bias of the biased variant (may be NULL)
  const float* b2;   // [B, h, dh] output bias (may be NULL)
  int64_t T;
  int h, m, nkv;
  int S;             // seed-query pooling: seeds per head (the output rows of an item)
  int window;        // sliding window: keys t - window < t' <= t
  const int32_t* offsets;   // sliding window: device offsets (sample starts)
  float scale;       // s
  float scale_log2;  // s * log2(e)
};

template <int DH>
struct FwdCfg {
  static constexpr int BN = 128;
  static constexpr int CH = DH < 64 ? DH : 64;          // elements per swizzled row
  static constexpr int NCH = DH / CH;                   // chunks along dh
  static constexpr uint32_t ROWB = CH * 2;              // bytes per row (64 or 128)
  static constexpr uint32_t CHUNKB = 128 * ROWB;        // one [128 x CH] chunk
  static constexpr uint32_t TILEB = NCH * CHUNKB;       // 128 * DH * 2
  static constexpr uint32_t SW = DH < 64 ? kSw64 : kSw128;
  static constexpr uint32_t ATOM = 8 * ROWB;            // 8-row group stride
  static constexpr int QST = DH == 128 ? 1 : 2;         // Q stages (a stage = tiles A and B)
  static constexpr int NS = DH == 32 ? 16 : (DH == 64 ? 8 : 4);   // K/V ring slots
  static constexpr uint32_t COL_S = 0, COL_O = 256;     // + 128*X, + DH*X for tile X
  // dh <= 64: P_X has columns of its own, [384 + 64X, 448 + 64X); dh = 128: P_X
  // aliases the first 64 columns of S_X
  static constexpr bool P_SEP = DH <= 64;
  static constexpr uint32_t COL_P = P_SEP ? 384 : COL_S;  // + 64*X (P_SEP) or + 128*X
  // barrier slots (SFREE / PFREE: S read out of TMEM / P read by its PV
  // product; used by the dh <= 64 kernel only)
  static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_SFULL = 4, B_PFULL = 6, B_OFULL = 8,
                       B_OEMPTY = 10, B_DRAIN = 12, B_SFREE = 13, B_PFREE = 15,
                       B_KVFULL = 17, B_KVEMPTY = 17 + NS, NBAR = 17 + 2 * NS;
  static constexpr uint32_t OFF_Q = 0, OFF_KV = QST * 2 * TILEB;
  // O epilogue: per activation warp, 32 rows x 64 columns of bf16 (128 B rows)
  // to turn its rows into whole-line global stores
  static constexpr uint32_t OSTG_WARP = 32 * 128;
  static constexpr uint32_t OFF_OSTG = OFF_KV + NS * TILEB;
  static constexpr uint32_t OFF_CTL = OFF_OSTG + 8 * OSTG_WARP;   // barriers, TMEM slot, abort flag
  static constexpr uint32_t CTL_BYTES = 1024;
  static constexpr uint32_t SMEM_USED = 1024 + OFF_CTL + CTL_BYTES;
  static_assert(OFF_KV >= QST * 2 * TILEB && OFF_OSTG >= OFF_KV + NS * TILEB &&
                    OFF_CTL >= OFF_OSTG + 8 * OSTG_WARP,
                "shared-memory regions overlap");
  // at least 120 KB so that two CTAs never share an SM (each allocates all 512 TMEM columns)
  static constexpr uint32_t SMEM = SMEM_USED > 120u * 1024u ? SMEM_USED : 120u * 1024u;
  static_assert(SMEM <= 232448u, "exceeds the 227 KB of shared memory a CTA can have");
  static_assert(8 * NBAR + 8 <= CTL_BYTES, "control block too small");
};

__device__ __forceinline__ float silu_tanh(float s, float half_scale) {
  const float hx = s * half_scale;                 // x/2 with x = s * scale
  return fmaf(hx, tanh_approx(hx), hx);             // x/2 * (1 + tanh(x/2)) = x * logistic(x)
}

// Work item p = tiles 2p (A) and 2p+1 (B, absent past the end of the list).
struct Pair {
  Tile a, b;
  bool has_b, share;   // share: same (sample, head), so the K/V blocks are common
};
__device__ __forceinline__ Pair load_pair(const Tile* tiles, int count, int p) {
  Pair r;
  r.a = tiles[2 * p];
  r.has_b = 2 * p + 1 < count;
  r.b = r.has_b ? tiles[2 * p + 1] : r.a;
  r.share = !r.has_b || (r.a.b == r.b.b && r.a.head == r.b.head);
  return r;
}

// Epilogue of one activation warp (TMEM lane quadrant `quad`, lane = tile
// row): its 32 O rows, times `inv`, rounded to bf16 and stored to row r <
// nrows of the tile at obase + r * row_stride.  The rows pass through the warp's own 4 KB of
// shared memory (`ostg`; 64 columns at a time, 16-byte chunks swizzled by
// row) so that every global store instruction writes whole rows: CPR lanes
// per row, 32 / CPR rows per instruction.  Arrives on `oempty` (the O
// accumulator is free) right after the last TMEM read, before the stores.
// `b2row` (DH values, or NULL) is the output bias added to every row.
template <int DH>
__device__ __forceinline__ void store_o_rows(uint32_t my_o, uint32_t ostg, float inv, int nrows,
                                             int quad, int lane, __nv_bfloat16* obase,
                                             int64_t row_stride, uint32_t oempty,
                                             const float* b2row = nullptr) {
  constexpr int PC = DH < 64 ? DH : 64;           // columns per pass
  constexpr int CPR = PC / 8;                     // 16-byte chunks per row
  constexpr int RPI = 32 / CPR;                   // rows per store instruction
  auto chunk_addr = [&](int r, int j) -> uint32_t {
    const int sw = CPR == 8 ? (r & 7) : ((r >> 1) & 3);
    return ostg + (uint32_t)(r * CPR * 16) + ((uint32_t)(j ^ sw) << 4);
  };
  const int rl = lane / CPR, jl = lane % CPR;      // read-back: row in group, chunk
#pragma unroll
  for (int c0 = 0; c0 < DH; c0 += PC) {
    uint32_t v[PC];
#pragma unroll
    for (int c = 0; c < PC; c += 16)
      tmem_ld_x16(my_o + c0 + c, *reinterpret_cast<uint32_t(*)[16]>(&v[c]));
    tmem_wait_ld();
    if (c0 + PC == DH) {
      tc_fence_before();
      mbar_arrive(oempty);                        // the O accumulator is free
    }
    if (b2row) {
#pragma unroll
      for (int c = 0; c < PC; ++c)
        v[c] = __float_as_uint(fmaf(__uint_as_float(v[c]), inv, __ldg(b2row + c0 + c)));
    } else {
#pragma unroll
      for (int c = 0; c < PC; ++c) v[c] = __float_as_uint(__uint_as_float(v[c]) * inv);
    }
#pragma unroll
    for (int j = 0; j < CPR; ++j) {
      const uint32_t p0 = pack_bf16x2(__uint_as_float(v[8 * j]), __uint_as_float(v[8 * j + 1]));
      const uint32_t p1 = pack_bf16x2(__uint_as_float(v[8 * j + 2]), __uint_as_float(v[8 * j + 3]));
      const uint32_t p2 = pack_bf16x2(__uint_as_float(v[8 * j + 4]), __uint_as_float(v[8 * j + 5]));
      const uint32_t p3 = pack_bf16x2(__uint_as_float(v[8 * j + 6]), __uint_as_float(v[8 * j + 7]));
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(chunk_addr(lane, j)),
                   "r"(p0), "r"(p1), "r"(p2), "r"(p3)
                   : "memory");
    }
    __syncwarp();
#pragma unroll
    for (int it = 0; it < CPR; ++it) {
      const int r = it * RPI + rl;                  // row within this warp's 32
      uint4 val;
      asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                   : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                   : "r"(chunk_addr(r, jl)));
      const int tr = quad * 32 + r;                 // tile row
      if (tr < nrows) *reinterpret_cast<uint4*>(obase + (int64_t)tr * row_stride + c0 + jl * 8) = val;
    }
    __syncwarp();
  }
}

// KEYMASK = false: every key block is full (m a multiple of 128), so the
// softmax carries no key mask.
template <int DH, int PHI, bool BIAS, bool KEYMASK = true>
__global__ void __launch_bounds__(kThreads, 1)
gdpa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<DH>;
  static_assert(!C::P_SEP, "dh <= 64 runs gdpa_fwd_early_kernel");
  constexpr bool SOFTMAX = PHI == GDPA_PHI_SOFTMAX;
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t IDESC_O = idesc_bf16(128, DH, 0, 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q;
  const uint32_t sKV = base + C::OFF_KV;
  uint8_t* ctl = gbase + C::OFF_CTL;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_QFULL + i), 1);
      mbar_init(bar(C::B_QEMPTY + i), 1);
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 128);
      mbar_init(bar(C::B_OFULL + i), 1);
      mbar_init(bar(C::B_OEMPTY + i), 128);
    }
    mbar_init(bar(C::B_DRAIN), 1);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar(C::B_KVFULL + i), 1);
      mbar_init(bar(C::B_KVEMPTY + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
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
  const int count = a.ws->tile_count;
  const int npairs = (count + 1) >> 1;
  const int nkv = a.nkv;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t ic = 0, slot = 0, sphase = 0;
      bool ok = true;
      auto load_kv = [&](const CUtensorMap* map, const Tile& tl, int j) -> bool {
        if (!mbar_wait(bar(C::B_KVEMPTY + slot), sphase ^ 1u, abort_flag, kTimeoutNs)) return false;
        mbar_expect_tx(bar(C::B_KVFULL + slot), C::TILEB);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c)
          tma_load_4d(sKV + slot * C::TILEB + c * C::CHUNKB, map, bar(C::B_KVFULL + slot),
                      c * C::CH, j * C::BN, tl.head, tl.b);
        if (++slot == (uint32_t)C::NS) {
          slot = 0;
          sphase ^= 1u;
        }
        return true;
      };
      for (int p = blockIdx.x; ok && p < npairs; p += gridDim.x, ++ic) {
        const Pair pr = load_pair(a.tiles, count, p);
        const uint32_t qs = ic % C::QST, qph = (ic / C::QST) & 1u;
        if (!mbar_wait(bar(C::B_QEMPTY + qs), qph ^ 1u, abort_flag, kTimeoutNs)) break;
        const uint32_t qaddr = sQ + qs * 2 * C::TILEB;
        mbar_expect_tx(bar(C::B_QFULL + qs), (pr.has_b ? 2u : 1u) * C::TILEB);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          tma_load_3d(qaddr + c * C::CHUNKB, &tmQ, bar(C::B_QFULL + qs), c * C::CH, pr.a.head,
                      pr.a.row0);
          if (pr.has_b)
            tma_load_3d(qaddr + C::TILEB + c * C::CHUNKB, &tmQ, bar(C::B_QFULL + qs), c * C::CH,
                        pr.b.head, pr.b.row0);
        }
        // K/V blocks in the order of their first use by the MMA issuer
        if (pr.share) {
          for (int j = 0; ok && j < nkv; ++j)
            ok = load_kv(&tmK, pr.a, j) && load_kv(&tmV, pr.a, j);
        } else {
          ok = load_kv(&tmK, pr.a, 0) && load_kv(&tmK, pr.b, 0);
          for (int j = 0; ok && j < nkv; ++j) {
            ok = load_kv(&tmV, pr.a, j);
            if (ok && j + 1 < nkv) ok = load_kv(&tmK, pr.a, j + 1);
            if (ok) ok = load_kv(&tmV, pr.b, j);
            if (ok && j + 1 < nkv) ok = load_kv(&tmK, pr.b, j + 1);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t ic = 0, slot = 0, sphase = 0;
      uint32_t pc[2] = {0u, 0u};   // PV groups issued per tile slot (P barrier phase)
      uint32_t oc[2] = {0u, 0u};   // items finished per tile slot (O barrier phase)
      bool ok = true;
      // next K/V ring slot, in the producer's load order
      auto take = [&]() -> int {
        if (!mbar_wait(bar(C::B_KVFULL + slot), sphase, abort_flag, kTimeoutNs)) return -1;
        tc_fence_after();
        const int s = (int)slot;
        if (++slot == (uint32_t)C::NS) {
          slot = 0;
          sphase ^= 1u;
        }
        return s;
      };
      for (int p = blockIdx.x; ok && p < npairs; p += gridDim.x, ++ic) {
        const Pair pr = load_pair(a.tiles, count, p);
        const uint32_t qs = ic % C::QST, qph = (ic / C::QST) & 1u;
        if (!mbar_wait(bar(C::B_QFULL + qs), qph, abort_flag, kTimeoutNs)) break;
        tc_fence_after();
        const uint32_t qbase = sQ + qs * 2 * C::TILEB;
        const int last_x = pr.has_b ? 1 : 0;
        const bool sep = !pr.share;              // A and B each have their own K/V slots
        // S_X(j) = Q_X K^T into S_X; the last S of the pair frees the Q stage
        auto issue_s = [&](int x, int ks, int j) {
          // descriptors built once per group: between two MMAs (whose issue waits
          // for the tensor core) only a constant add remains
          const uint64_t a0 = smem_desc(qbase + x * C::TILEB, 16, C::ATOM, C::SW);
          const uint64_t b0 = smem_desc(sKV + ks * C::TILEB, 16, C::ATOM, C::SW);
          const uint32_t dcol = tmem + C::COL_S + 128 * x;
#pragma unroll
          for (int k = 0; k < DH / 16; ++k) {
            const uint32_t off = (k / (C::CH / 16)) * C::CHUNKB + (k % (C::CH / 16)) * 32;
            mma_ss(dcol, desc_advance(a0, off), desc_advance(b0, off), IDESC_S, k > 0 ? 1u : 0u);
          }
          mma_commit(bar(C::B_SFULL + x));
          if (x == last_x && j == nkv - 1) mma_commit(bar(C::B_QEMPTY + qs));
        };
        // O_X += P_X(j) V_j once the activation group has written P_X(j)
        auto issue_pv = [&](int x, int vs, int j) -> bool {
          if (!mbar_wait(bar(C::B_PFULL + x), pc[x] & 1u, abort_flag, kTimeoutNs)) return false;
          ++pc[x];
          if (j == 0 && !mbar_wait(bar(C::B_OEMPTY + x), (oc[x] & 1u) ^ 1u, abort_flag, kTimeoutNs))
            return false;
          tc_fence_after();
          const uint64_t v0 = smem_desc(sKV + vs * C::TILEB, C::CHUNKB, C::ATOM, C::SW);
          const uint32_t ocol = tmem + C::COL_O + DH * x;
          const uint32_t pcol = tmem + C::COL_P + (C::P_SEP ? 64 : 128) * x;
          const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
          for (int k = 0; k < C::BN / 16; ++k)
            mma_ts(ocol, pcol + k * 8, desc_advance(v0, k * 2 * C::ATOM), IDESC_O, k > 0 ? 1u : acc0);
          if (j == nkv - 1) {
            mma_commit(bar(C::B_OFULL + x));
            ++oc[x];
          }
          return true;
        };
        auto release = [&](int s) { mma_commit(bar(C::B_KVEMPTY + s)); };

        int ka = take();
        if (ka < 0) break;
        issue_s(0, ka, 0);
        if (!pr.has_b || sep) release(ka);
        if (pr.has_b) {
          const int kb = sep ? take() : ka;
          if (kb < 0) break;
          issue_s(1, kb, 0);
          release(kb);
        }
        for (int j = 0; ok && j < nkv; ++j) {
          const int va = take();
          if (va < 0 || !issue_pv(0, va, j)) {
            ok = false;
            break;
          }
          if (!pr.has_b || sep) release(va);
          int kn = -1;
          if (j + 1 < nkv) {
            kn = take();
            if (kn < 0) {
              ok = false;
              break;
            }
            issue_s(0, kn, j + 1);
            if (!pr.has_b || sep) release(kn);
          }
          if (pr.has_b) {
            const int vb = sep ? take() : va;
            if (vb < 0 || !issue_pv(1, vb, j)) {
              ok = false;
              break;
            }
            release(vb);
            if (j + 1 < nkv) {
              const int kb = sep ? take() : kn;
              if (kb < 0) {
                ok = false;
                break;
              }
              issue_s(1, kb, j + 1);
              release(kb);
            }
          }
        }
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ activation groups
    const int grp = (warp - 4) >> 2;            // tile slot: 0 = A, 1 = B
    const int quad = warp & 3;                  // TMEM lane quadrant
    const int row = quad * 32 + lane;           // tile row owned by this thread
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t my_s = tmem + lane_off + C::COL_S + 128 * grp;
    const uint32_t my_o = tmem + lane_off + C::COL_O + DH * grp;
    const uint32_t my_p = tmem + lane_off + C::COL_P + (C::P_SEP ? 64 : 128) * grp;
    const float c2 = a.scale_log2;
    const float half_scale = 0.5f * a.scale;
    uint32_t sc = 0, oc = 0;
    bool ok = true;
    for (int p = blockIdx.x; ok && p < npairs; p += gridDim.x) {
      const Pair pr = load_pair(a.tiles, count, p);
      if (grp == 1 && !pr.has_b) continue;
      const Tile tl = grp ? pr.b : pr.a;
      float m_run = -INFINITY, l_run = 0.f;
      int steps = 0;
      // biased variant: the key bias of each block passes through the first
      // 512 B of this warp's epilogue staging area, pre-multiplied for the
      // activation (log2 e for softmax, 1/2 for SiLU); the logits are then
      // biased right after each TMEM read (the activation takes mul = 1)
      const float* b1row =
          BIAS && a.b1 ? a.b1 + ((int64_t)tl.b * a.h + tl.head) * a.m : nullptr;
      const uint32_t bstg = base + C::OFF_OSTG + (uint32_t)(warp - 4) * C::OSTG_WARP;
      constexpr float kBiasMul =
          SOFTMAX ? 1.4426950408889634f : (PHI == GDPA_PHI_SILU ? 0.5f : 1.f);
      const float bmul = SOFTMAX ? c2 : (PHI == GDPA_PHI_SILU ? half_scale : a.scale);
      // s[0..n) := s * bmul + b1 of columns col0.. (from the staging area)
      auto bias_cols = [&](uint32_t* sv, int n, int col0) {
#pragma unroll
        for (int i = 0; i < n; i += 4) {
          float4 b4;
          asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                       : "=f"(b4.x), "=f"(b4.y), "=f"(b4.z), "=f"(b4.w)
                       : "r"(bstg + 4 * (col0 + i)));
          sv[i] = __float_as_uint(fmaf(__uint_as_float(sv[i]), bmul, b4.x));
          sv[i + 1] = __float_as_uint(fmaf(__uint_as_float(sv[i + 1]), bmul, b4.y));
          sv[i + 2] = __float_as_uint(fmaf(__uint_as_float(sv[i + 2]), bmul, b4.z));
          sv[i + 3] = __float_as_uint(fmaf(__uint_as_float(sv[i + 3]), bmul, b4.w));
        }
      };
      const float c2e = BIAS ? 1.f : c2;          // softmax multiplier after the bias pass
      for (int j = 0; j < nkv; ++j, ++sc) {
        if constexpr (BIAS) {
          float bl[4] = {0.f, 0.f, 0.f, 0.f};
          if (b1row) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int key = j * C::BN + 4 * lane + u;
              bl[u] = key < a.m ? __ldg(b1row + key) * kBiasMul : 0.f;
            }
          }
          __syncwarp();
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(bstg + 16 * lane),
                       "f"(bl[0]), "f"(bl[1]), "f"(bl[2]), "f"(bl[3])
                       : "memory");
          __syncwarp();
        }
        bool w = mbar_wait(bar(C::B_SFULL + grp), sc & 1u, abort_flag, kTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int valid = min(C::BN, a.m - j * C::BN);
        if constexpr (SOFTMAX) {
          // The row is handled in two 64-column halves read from TMEM, so at most
          // 64 logits and the 64 packed P words are live at once.
          // Row offset m_run (log2 units): the first key block of a tile takes the
          // exact row max.  Later blocks reuse m_run as long as every
          // p = 2^(x - m_run) stays <= 2^8, which a row sum <= 2^8 guarantees;
          // otherwise (or on overflow, where the sum is not finite) the exact max
          // of this block is taken and m_run moves when it grew by more than 2^8.
          // Softmax does not depend on the offset, so this only skips the max.
          uint32_t sh[64];
          auto load_half = [&](int hf) {
            tmem_ld_x32(my_s + 64 * hf, *reinterpret_cast<uint32_t(*)[32]>(&sh[0]));
            tmem_ld_x32(my_s + 64 * hf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sh[32]));
            tmem_wait_ld();
            if constexpr (BIAS) bias_cols(sh, 64, 64 * hf);
          };
          auto row_max = [&]() -> float {
            float m8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = c2e >= 0.f ? -INFINITY : INFINITY;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              load_half(hf);
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                const float x = __uint_as_float(sh[i]);
                if (!KEYMASK || valid == C::BN || 64 * hf + i < valid)
                  m8[i & 7] = c2e >= 0.f ? fmaxf(m8[i & 7], x) : fminf(m8[i & 7], x);
              }
            }
#pragma unroll
            for (int u = 4; u > 0; u >>= 1)
#pragma unroll
              for (int v = 0; v < u; ++v)
                m8[v] = c2e >= 0.f ? fmaxf(m8[v], m8[v + u]) : fminf(m8[v], m8[v + u]);
            return m8[0] * c2e;
          };
          uint32_t pk[64];
          auto exp_pack = [&]() -> float {
            const float neg_m = -m_run;
            float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              load_half(hf);
              uint32_t* pkh = pk + 32 * hf;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int col = 64 * hf + 2 * i;
                float p0 = ex2_approx(fmaf(__uint_as_float(sh[2 * i]), c2e, neg_m));
                float p1 = ex2_approx(fmaf(__uint_as_float(sh[2 * i + 1]), c2e, neg_m));
                if (KEYMASK && valid < C::BN) {
                  p0 = col < valid ? p0 : 0.f;
                  p1 = col + 1 < valid ? p1 : 0.f;
                }
                rs8[(2 * i) & 7] += p0;
                rs8[(2 * i + 1) & 7] += p1;
                pkh[i] = pack_bf16x2(p0, p1);
              }
            }
            return ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
          };
          float alpha = 1.f, rs = 0.f;
          bool resc = false;
          // pass 0: the first key block of the tile takes the exact max, later
          // blocks reuse m_run; pass 1 (rare) redoes the block with the exact max
#pragma unroll 1
          for (int pass = 0; pass < 2; ++pass) {
            const bool need_max = pass == 0 ? steps == 0 : !(rs <= 256.f);
            if (__any_sync(0xffffffffu, need_max)) {
              const float m_new = row_max();
              if (need_max) {
                if (pass == 0) {
                  m_run = m_new;
                } else if (m_new > m_run + 8.0f) {
                  alpha = ex2_approx(m_run - m_new);
                  m_run = m_new;
                  resc = true;
                }
              }
            }
            rs = exp_pack();
            if (pass == 1 || steps == 0 || !__any_sync(0xffffffffu, !(rs <= 256.f))) break;
          }
          // P aliases the first 64 columns of S
          tmem_st_x32(my_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
          tmem_st_x32(my_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
          l_run = l_run * alpha + rs;
          if (__any_sync(0xffffffffu, resc)) {
            #pragma unroll
            for (int c = 0; c < DH; c += 16) {
              uint32_t ov[16];
              tmem_ld_x16(my_o + c, ov);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              tmem_st_x16(my_o + c, ov);
            }
          }
          tmem_wait_st();
        } else {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t s[32];
            tmem_ld_x32(my_s + 32 * c, s);
            tmem_wait_ld();
            if constexpr (BIAS) bias_cols(s, 32, 32 * c);
            // BIAS: s already holds the biased logit (SiLU: its half)
            const float sm = BIAS ? 1.f : a.scale, hsm = BIAS ? 1.f : half_scale;
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0 = __uint_as_float(s[2 * i]), x1 = __uint_as_float(s[2 * i + 1]);
              float p0, p1;
              if constexpr (PHI == GDPA_PHI_SILU) {
                p0 = silu_tanh(x0, hsm);
                p1 = silu_tanh(x1, hsm);
              } else if constexpr (PHI == GDPA_PHI_RELU) {
                p0 = relu_f(x0 * sm);
                p1 = relu_f(x1 * sm);
              } else if constexpr (PHI == GDPA_PHI_GELU) {
                p0 = gelu_f(x0 * sm);
                p1 = gelu_f(x1 * sm);
              } else {
                p0 = x0 * sm;
                p1 = x1 * sm;
              }
              pk[i] = pack_bf16x2(p0, p1);
            }
            tmem_st_x16(my_p + 16 * c, pk);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + grp));
        ++steps;
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      bool w = mbar_wait(bar(C::B_OFULL + grp), oc & 1u, abort_flag, kTimeoutNs);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = SOFTMAX ? 1.f / l_run : 1.f;
      const bool store = row < tl.rows;
      store_o_rows<DH>(my_o, base + C::OFF_OSTG + (uint32_t)(warp - 4) * C::OSTG_WARP, inv,
                       tl.rows, quad, lane, a.o + ((int64_t)tl.row0 * a.h + tl.head) * DH,
                       (int64_t)a.h * DH, bar(C::B_OEMPTY + grp),
                       BIAS && a.b2 ? a.b2 + ((int64_t)tl.b * a.h + tl.head) * DH : nullptr);
      if (SOFTMAX && store && a.lse != nullptr)
        a.lse[(int64_t)tl.head * a.T + tl.row0 + row] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      ++oc;
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    report(a.ws, GDPA_ERR_TIMEOUT);
    volatile int never = 0;
    if (warp == 1 && lane == 0) {
      mma_commit(bar(C::B_DRAIN));                       // all MMAs issued so far
      mbar_wait(bar(C::B_DRAIN), 0, &never, kTimeoutNs);
    }
    if (warp == 0 && lane == 0) {                         // let in-flight TMA loads land
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

// ---------------------------------------------------------------------------
// dh <= 64: S released early.
//
// P_X has TMEM columns of its own, so S_X is free as soon as the activation
// group has read it into registers.  The group arrives on SFREE_X right after
// that read, and the MMA issuer queues S_X(j+1) ahead of PV_X(j) (and, at the
// last key block of an item, the next item's S_X(0)): the tensor core computes
// the next logits while the activation of this block runs, and the activation
// finds its next S already in TMEM.  P_X is rewritten only after PFREE_X
// reports that the previous PV_X has read it.
//
// Softmax takes the exact row maximum of every key block from registers
// (three-input max), keeps the running offset while the block maximum stays
// within 2^8 of it and otherwise moves it and rescales O (rare).  A fixed
// share of the exp2 evaluations (kPolyPairs of every 8 pairs of columns) runs
// on the FMA pipe (exp2_fma2) instead of the MUFU unit, which the exp2 and the
// bf16 packs keep the busiest pipe of the dh = 64 forward: one transcendental
// per logit against 4 * dh = 256 tensor FLOPs per logit.  Two of eight
// measured 2.5% faster than none on the power-law softmax forward; three of
// eight slower (the FMA and ALU work of the polynomial).
//
// Registers: the launch gives 168 per thread (384 x 168 = 64,512); warps 0-3
// drop to 80 and the two activation warpgroups rise to 208 (a thread holds a
// whole 128-column S row): 128 x 80 + 256 x 208 = 63,488 <= 64,512.
constexpr int kPolyPairs = 2;

// Modes of the dh <= 64 forward kernel: the GDPA operator, seed-query pooling
// (first level of HSP) and sliding-window self-attention on the jagged tokens.
constexpr int kModeGdpa = 0, kModePool = 1, kModeWindow = 2;

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// The row's largest (NEG: smallest) raw logit over 128 columns.
template <bool NEG>
__device__ __forceinline__ float row_extreme(const uint32_t (&s)[128]) {
  float e[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) e[u] = __uint_as_float(s[u]);
#pragma unroll
  for (int i = 4; i < 128; i += 8) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float a0 = __uint_as_float(s[i + 2 * u]), a1 = __uint_as_float(s[i + 2 * u + 1]);
      e[u] = NEG ? fmin3(e[u], a0, a1) : fmax3(e[u], a0, a1);
    }
  }
  return NEG ? fmin3(fminf(e[0], e[1]), e[2], e[3]) : fmax3(fmaxf(e[0], e[1]), e[2], e[3]);
}

// KEYMASK = false: every key block is full (GDPA with m a multiple of 128),
// so the softmax needs no key mask and the kernel carries none.
template <int DH, int PHI, bool BIAS, int MODE, bool KEYMASK = true>
__global__ void __launch_bounds__(kThreads, 1)
gdpa_fwd_early_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<DH>;
  static_assert(C::P_SEP, "needs P in TMEM columns of its own");
  constexpr bool POOL = MODE == kModePool, WIN = MODE == kModeWindow;
  static_assert(MODE == kModeGdpa || (PHI == GDPA_PHI_SOFTMAX && !BIAS),
                "pooling and sliding-window attention are softmax attention");
  constexpr bool SOFTMAX = PHI == GDPA_PHI_SOFTMAX;
  constexpr uint32_t IDESC_S = idesc_bf16(128, 128, 0, 0);
  constexpr uint32_t IDESC_O = idesc_bf16(128, DH, 0, 1);

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const uint32_t sQ = base + C::OFF_Q;
  const uint32_t sKV = base + C::OFF_KV;
  uint8_t* ctl = gbase + C::OFF_CTL;
  const uint32_t bar0 = smem_u32(ctl);
  auto bar = [&](int i) -> uint32_t { return bar0 + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * C::NBAR);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 8 * C::NBAR + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(C::B_QFULL + i), 1);
      mbar_init(bar(C::B_QEMPTY + i), 2);      // both issuers' last S of an item
      mbar_init(bar(C::B_SFULL + i), 1);
      mbar_init(bar(C::B_PFULL + i), 128);
      mbar_init(bar(C::B_OFULL + i), 1);
      mbar_init(bar(C::B_OEMPTY + i), 128);
      mbar_init(bar(C::B_SFREE + i), 128);
      mbar_init(bar(C::B_PFREE + i), 1);
    }
    mbar_init(bar(C::B_DRAIN), 2);
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(bar(C::B_KVFULL + i), 1);
      mbar_init(bar(C::B_KVEMPTY + i), 2);     // two releases per load (see the issuers)
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmQ);
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
  const int count = a.ws->tile_count;
  const int stride = gridDim.x;
  // GDPA: work item p = query tiles 2p, 2p+1 of the jagged tile list, all with
  // a.nkv key blocks of a.m keys.  Seed-query pooling (POOL): item p = heads
  // (2k, 2k+1) of one sample, the seeds of each head as the 128-row query
  // tile, the sample's n_b tokens as ceil(n_b / 128) key blocks.  Sliding
  // window (WIN): item p = heads (2k, 2k+1) of one 128-row query tile; its
  // keys are the sample's tokens from kstart = max(sample start, row0 - w + 1)
  // to the tile's last row, masked per element to the causal window.
  const int npairs = MODE == kModeGdpa ? (count + 1) >> 1 : count;
  auto get_pair = [&](int p) -> Pair {
    if constexpr (MODE != kModeGdpa) {
      Pair r;
      r.a = a.tiles[p];
      if (WIN) r.a.head *= 2;                        // the list holds head pairs
      r.has_b = r.a.head + 1 < a.h;
      r.b = r.a;
      r.b.head = r.a.head + 1;
      r.share = !r.has_b;     // a lone head streams its K/V once, like a shared pair
      return r;
    } else {
      return load_pair(a.tiles, count, p);
    }
  };
  // first key row of a window item (WIN only)
  auto win_kstart = [&](const Tile& t) -> int {
    const int lo = t.row0 - a.window + 1, s0 = __ldg(a.offsets + t.b);
    return lo > s0 ? lo : s0;
  };
  auto pair_nkv = [&](const Pair& pr) -> int {
    if constexpr (POOL) return (pr.a.rows + 127) >> 7;
    if constexpr (WIN) return (pr.a.row0 + pr.a.rows - win_kstart(pr.a) + 127) >> 7;
    return a.nkv;
  };

  if (warp < 4) {
    setmaxnreg_dec<80>();
    if (warp == 0 && lane == 0) {
      // ---------------------------------------------------------- producer
      // Load order = the MMA issuer's order of first use: Q and K(0) of the
      // first item; then per key block j: K(j+1) (or, at the last block, the
      // next item's Q and K(0)), V(j).  Tiles A and B of a pair that share
      // their (sample, head) share each K/V load.
      uint32_t slot = 0, sphase = 0;
      auto load_kv = [&](const CUtensorMap* map, const Tile& tl, int j) -> bool {
        if (!mbar_wait(bar(C::B_KVEMPTY + slot), sphase ^ 1u, abort_flag, kTimeoutNs)) return false;
        mbar_expect_tx(bar(C::B_KVFULL + slot), C::TILEB);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          if constexpr (MODE != kModeGdpa)   // tokens [T, h, dh], masked later
            tma_load_3d(sKV + slot * C::TILEB + c * C::CHUNKB, map, bar(C::B_KVFULL + slot),
                        c * C::CH, tl.head, (WIN ? win_kstart(tl) : tl.row0) + j * C::BN);
          else
            tma_load_4d(sKV + slot * C::TILEB + c * C::CHUNKB, map, bar(C::B_KVFULL + slot),
                        c * C::CH, j * C::BN, tl.head, tl.b);
        }
        if (++slot == (uint32_t)C::NS) {
          slot = 0;
          sphase ^= 1u;
        }
        return true;
      };
      auto load_both = [&](const CUtensorMap* map, const Pair& pr, int j) -> bool {
        if (!load_kv(map, pr.a, j)) return false;
        return pr.share ? true : load_kv(map, pr.b, j);
      };
      auto load_q = [&](const Pair& pr, uint32_t ic) -> bool {
        const uint32_t qs = ic % C::QST, qph = (ic / C::QST) & 1u;
        if (!mbar_wait(bar(C::B_QEMPTY + qs), qph ^ 1u, abort_flag, kTimeoutNs)) return false;
        const uint32_t qaddr = sQ + qs * 2 * C::TILEB;
        mbar_expect_tx(bar(C::B_QFULL + qs), (pr.has_b ? 2u : 1u) * C::TILEB);
#pragma unroll
        for (int c = 0; c < C::NCH; ++c) {
          if constexpr (POOL) {   // seeds [h, S, dh] of heads a, b; rows >= S read as zero
            tma_load_3d(qaddr + c * C::CHUNKB, &tmQ, bar(C::B_QFULL + qs), c * C::CH, 0,
                        pr.a.head);
            if (pr.has_b)
              tma_load_3d(qaddr + C::TILEB + c * C::CHUNKB, &tmQ, bar(C::B_QFULL + qs),
                          c * C::CH, 0, pr.b.head);
          } else {
            tma_load_3d(qaddr + c * C::CHUNKB, &tmQ, bar(C::B_QFULL + qs), c * C::CH, pr.a.head,
                        pr.a.row0);
            if (pr.has_b)
              tma_load_3d(qaddr + C::TILEB + c * C::CHUNKB, &tmQ, bar(C::B_QFULL + qs),
                          c * C::CH, pr.b.head, pr.b.row0);
          }
        }
        return true;
      };
      int p = blockIdx.x;
      bool ok = p < npairs;
      if (ok) {
        const Pair pr = get_pair(p);
        ok = load_q(pr, 0) && load_both(&tmK, pr, 0);
      }
      for (uint32_t ic = 0; ok && p < npairs; p += stride, ++ic) {
        const Pair pr = get_pair(p);
        const int nkv = pair_nkv(pr);
        const bool has_next = p + stride < npairs;
        for (int j = 0; ok && j < nkv; ++j) {
          if (j + 1 < nkv) {
            ok = load_both(&tmK, pr, j + 1);
          } else if (has_next) {
            const Pair pn = get_pair(p + stride);
            ok = load_q(pn, ic + 1) && load_both(&tmK, pn, 0);
          }
          if (ok) ok = load_both(&tmV, pr, j);
        }
      }
    } else if ((warp == 1 || warp == 3) && lane == 0) {
      // ---------------------------------------------------------- MMA issuers
      // One issuer per tile slot x (warp 1: A, warp 3: B), so that neither
      // tile's products wait behind the other's in one in-order stream.  Both
      // replay the producer's load order to find the ring slot of each of
      // their K/V blocks.  Every load is released twice on KVEMPTY: once by
      // each issuer when A and B share it, else twice by its one reader.  The
      // Q stage of an item is released twice on QEMPTY the same way.
      const int x = warp == 1 ? 0 : 1;
      uint32_t seq = 0;                 // ring loads replayed so far
      uint32_t s_cnt = 0, pv_cnt = 0, o_cnt = 0;
      bool ok = true;
      auto replay = [&](const Pair& pr) -> uint32_t {   // load_both: this tile's load index
        const uint32_t ia = seq++;
        const uint32_t ib = pr.share ? ia : seq++;
        return x == 0 ? ia : ib;
      };
      auto mine = [&](const Pair& pr) { return x == 0 || pr.has_b; };
      auto releases = [&](const Pair& pr) -> int { return pr.has_b && pr.share ? 1 : 2; };
      auto wait_load = [&](uint32_t idx) -> bool {
        if (!mbar_wait(bar(C::B_KVFULL + (int)(idx % C::NS)), (idx / C::NS) & 1u, abort_flag,
                       kTimeoutNs))
          return false;
        tc_fence_after();
        return true;
      };
      auto release = [&](uint32_t idx, int n) {
        for (int r = 0; r < n; ++r) mma_commit(bar(C::B_KVEMPTY + (int)(idx % C::NS)));
      };
      // S_x = Q_x K^T once the group has read the previous S_x out of TMEM;
      // the last S of an item releases its Q stage.
      auto issue_s = [&](const Pair& pr, uint32_t qs, uint32_t kidx, bool last) -> bool {
        if (!wait_load(kidx)) return false;
        if (s_cnt > 0 &&
            !mbar_wait(bar(C::B_SFREE + x), (s_cnt - 1) & 1u, abort_flag, kTimeoutNs))
          return false;
        ++s_cnt;
        tc_fence_after();
        const int ks = (int)(kidx % C::NS);
        const uint64_t a0 = smem_desc(sQ + qs * 2 * C::TILEB + x * C::TILEB, 16, C::ATOM, C::SW);
        const uint64_t b0 = smem_desc(sKV + ks * C::TILEB, 16, C::ATOM, C::SW);
        const uint32_t dcol = tmem + C::COL_S + 128 * x;
#pragma unroll
        for (int k = 0; k < DH / 16; ++k) {
          const uint32_t off = (k / (C::CH / 16)) * C::CHUNKB + (k % (C::CH / 16)) * 32;
          mma_ss(dcol, desc_advance(a0, off), desc_advance(b0, off), IDESC_S, k > 0 ? 1u : 0u);
        }
        mma_commit(bar(C::B_SFULL + x));
        if (last) {
          mma_commit(bar(C::B_QEMPTY + qs));
          if (!pr.has_b) mma_commit(bar(C::B_QEMPTY + qs));
        }
        release(kidx, releases(pr));
        return true;
      };
      // O_x += P_x V once the group has written P_x; PFREE_x reports that P_x
      // has been read, OFULL_x (last key block) that O_x is complete.
      auto issue_pv = [&](const Pair& pr, uint32_t vidx, int j, int nkv) -> bool {
        if (!wait_load(vidx)) return false;
        if (!mbar_wait(bar(C::B_PFULL + x), pv_cnt & 1u, abort_flag, kTimeoutNs)) return false;
        ++pv_cnt;
        if (j == 0 &&
            !mbar_wait(bar(C::B_OEMPTY + x), (o_cnt & 1u) ^ 1u, abort_flag, kTimeoutNs))
          return false;
        tc_fence_after();
        const int vs = (int)(vidx % C::NS);
        const uint64_t v0 = smem_desc(sKV + vs * C::TILEB, C::CHUNKB, C::ATOM, C::SW);
        const uint32_t ocol = tmem + C::COL_O + DH * x;
        const uint32_t pcol = tmem + C::COL_P + 64 * x;
        const uint32_t acc0 = j > 0 ? 1u : 0u;
#pragma unroll
        for (int k = 0; k < C::BN / 16; ++k)
          mma_ts(ocol, pcol + k * 8, desc_advance(v0, k * 2 * C::ATOM), IDESC_O, k > 0 ? 1u : acc0);
        mma_commit(bar(C::B_PFREE + x));
        if (j == nkv - 1) {
          mma_commit(bar(C::B_OFULL + x));
          ++o_cnt;
        }
        release(vidx, releases(pr));
        return true;
      };
      int p = blockIdx.x;
      uint32_t k0 = 0;                   // this tile's K(0) load of item p
      bool s0_done = false;              // S_x(0) of item p already issued
      if (p < npairs) k0 = replay(get_pair(p));
      for (uint32_t ic = 0; ok && p < npairs; p += stride, ++ic) {
        const Pair pr = get_pair(p);
        const int nkv = pair_nkv(pr);
        const uint32_t qs = ic % C::QST, qph = (ic / C::QST) & 1u;
        const bool has_next = p + stride < npairs;
        const bool me = mine(pr);
        if (me && !s0_done)
          ok = mbar_wait(bar(C::B_QFULL + qs), qph, abort_flag, kTimeoutNs) &&
               issue_s(pr, qs, k0, nkv == 1);
        s0_done = false;
        for (int j = 0; ok && j < nkv; ++j) {
          if (j + 1 < nkv) {
            const uint32_t kn = replay(pr);
            if (me) ok = issue_s(pr, qs, kn, j + 2 == nkv);
          } else if (has_next) {
            // the next item's first S, ahead of this item's last PV
            const Pair pn = get_pair(p + stride);
            k0 = replay(pn);
            if (mine(pn)) {
              const uint32_t qn = (ic + 1) % C::QST, qnph = ((ic + 1) / C::QST) & 1u;
              ok = mbar_wait(bar(C::B_QFULL + qn), qnph, abort_flag, kTimeoutNs) &&
                   issue_s(pn, qn, k0, pair_nkv(pn) == 1);
              s0_done = true;
            }
          }
          const uint32_t vi = replay(pr);
          if (ok && me) ok = issue_pv(pr, vi, j, nkv);
        }
      }
    }
  } else {
    setmaxnreg_inc<208>();
    // ------------------------------------------------------------ activation groups
    const int grp = (warp - 4) >> 2;            // tile slot: 0 = A, 1 = B
    const int quad = warp & 3;                  // TMEM lane quadrant
    const int row = quad * 32 + lane;           // tile row owned by this thread
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t my_s = tmem + lane_off + C::COL_S + 128 * grp;
    const uint32_t my_o = tmem + lane_off + C::COL_O + DH * grp;
    const uint32_t my_p = tmem + lane_off + C::COL_P + 64 * grp;
    const float c2 = a.scale_log2;
    const float2 c2v = make_float2(c2, c2);
    const float half_scale = 0.5f * a.scale;
    uint32_t sc = 0, oc = 0;
    bool ok = true;
    for (int p = blockIdx.x; ok && p < npairs; p += stride) {
      const Pair pr = get_pair(p);
      if (grp == 1 && !pr.has_b) continue;
      const Tile tl = grp ? pr.b : pr.a;
      const int nkv = pair_nkv(pr);
      const int kv_len = POOL ? tl.rows : a.m;          // keys of the item (not WIN)
      const int out_rows = POOL ? a.S : tl.rows;        // output rows of the item
      const int kstart = WIN ? win_kstart(tl) : 0;
      if (quad * 32 >= out_rows) {
        // every row of this warp lies past the tile's rows: those rows of O are
        // never stored, so the warp computes nothing and only keeps its part
        // in every barrier of the item
        for (int j = 0; j < nkv; ++j, ++sc) {
          bool w = mbar_wait(bar(C::B_SFULL + grp), sc & 1u, abort_flag, kTimeoutNs);
          if (sc > 0 && w) w = mbar_wait(bar(C::B_PFREE + grp), (sc - 1) & 1u, abort_flag, kTimeoutNs);
          if (!__all_sync(0xffffffffu, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          tc_fence_before();
          mbar_arrive(bar(C::B_SFREE + grp));
          mbar_arrive(bar(C::B_PFULL + grp));
        }
        if (!ok) break;
        const bool w = mbar_wait(bar(C::B_OFULL + grp), oc & 1u, abort_flag, kTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        ++oc;
        tc_fence_after();
        tc_fence_before();
        mbar_arrive(bar(C::B_OEMPTY + grp));
        continue;
      }
      float m_run = 0.f, l_run = 0.f;
      // biased variant: the key bias of each block passes through the first
      // 512 B of this warp's epilogue staging area (unused until the epilogue),
      // pre-multiplied for the activation (log2 e for softmax, 1/2 for SiLU)
      const float* b1row =
          BIAS && a.b1 ? a.b1 + ((int64_t)tl.b * a.h + tl.head) * a.m : nullptr;
      const uint32_t bstg = base + C::OFF_OSTG + (uint32_t)(warp - 4) * C::OSTG_WARP;
      constexpr float kBiasMul =
          SOFTMAX ? 1.4426950408889634f : (PHI == GDPA_PHI_SILU ? 0.5f : 1.f);
      for (int j = 0; j < nkv; ++j, ++sc) {
        float bl[4] = {0.f, 0.f, 0.f, 0.f};
        if (BIAS && b1row) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int key = j * C::BN + 4 * lane + u;
            bl[u] = key < a.m ? __ldg(b1row + key) * kBiasMul : 0.f;
          }
        }
        bool w = mbar_wait(bar(C::B_SFULL + grp), sc & 1u, abort_flag, kTimeoutNs);
        if (!__all_sync(0xffffffffu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t s[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld_x32(my_s + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&s[32 * c]));
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(bar(C::B_SFREE + grp));      // S_x may be overwritten now
        const int valid = min(C::BN, kv_len - j * C::BN);
        if constexpr (BIAS) {
          // s := s * mul + b1 (mul: s log2 e for softmax, s / 2 for SiLU, s
          // otherwise); the activation below then takes mul = 1
          __syncwarp();
          asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(bstg + 16 * lane),
                       "f"(bl[0]), "f"(bl[1]), "f"(bl[2]), "f"(bl[3])
                       : "memory");
          __syncwarp();
          const float mul = SOFTMAX ? c2 : (PHI == GDPA_PHI_SILU ? half_scale : a.scale);
          const float2 mulv = make_float2(mul, mul);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float4 b4;
            asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                         : "=f"(b4.x), "=f"(b4.y), "=f"(b4.z), "=f"(b4.w)
                         : "r"(bstg + 16 * i));
            const float2 y0 = __ffma2_rn(
                make_float2(__uint_as_float(s[4 * i]), __uint_as_float(s[4 * i + 1])), mulv,
                make_float2(b4.x, b4.y));
            const float2 y1 = __ffma2_rn(
                make_float2(__uint_as_float(s[4 * i + 2]), __uint_as_float(s[4 * i + 3])), mulv,
                make_float2(b4.z, b4.w));
            s[4 * i] = __float_as_uint(y0.x);
            s[4 * i + 1] = __float_as_uint(y0.y);
            s[4 * i + 2] = __float_as_uint(y1.x);
            s[4 * i + 3] = __float_as_uint(y1.y);
          }
        }
        uint32_t pk[64];
        float alpha = 1.f;
        bool resc = false;
        {
          if constexpr (SOFTMAX) {
            const bool neg = !BIAS && c2 < 0.f;
            // keys of this block that this row may see: columns [clo, chi]
            int clo = 0, chi = valid - 1;
            if constexpr (WIN) {
              const int kb0 = kstart + j * C::BN, qpos = tl.row0 + row;
              clo = max(0, qpos - a.window + 1 - kb0);
              chi = min(C::BN - 1, qpos - kb0);
            }
            const bool partial =
                KEYMASK && (WIN ? __any_sync(0xffffffffu, clo > 0 || chi < C::BN - 1)
                                : valid < C::BN);
            if (partial) {
              const uint32_t fill = __float_as_uint(neg ? INFINITY : -INFINITY);
#pragma unroll
              for (int i = 0; i < 128; ++i) s[i] = i >= clo && i <= chi ? s[i] : fill;
            }
            const float m_blk =
                (neg ? row_extreme<true>(s) : row_extreme<false>(s)) * (BIAS ? 1.f : c2);
            if (j == 0) {
              m_run = m_blk;
            } else if (m_blk > m_run + 8.f) {
              alpha = ex2_approx(m_run - m_blk);
              m_run = m_blk;
              resc = true;
            }
            // masked logits hold -inf (+inf for a negative scale), so their exp2 is
            // exactly 0; a row with no visible key yet keeps m_run = -inf and takes
            // offset 0 (its exponents are all -inf as well)
            const float mo = m_run == -INFINITY ? 0.f : -m_run;
            const float2 negm = make_float2(mo, mo);
            float2 acc[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const float2 x = __ffma2_rn(
                  make_float2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1])),
                  BIAS ? make_float2(1.f, 1.f) : c2v, negm);
              float2 e;
              if ((i & 7) < kPolyPairs) {
                e = exp2_fma2(x);
              } else {
                e.x = ex2_approx(x.x);
                e.y = ex2_approx(x.y);
              }
              acc[i & 3] = __fadd2_rn(acc[i & 3], e);
              pk[i] = pack_bf16x2(e.x, e.y);
            }
            const float2 r01 = __fadd2_rn(acc[0], acc[1]), r23 = __fadd2_rn(acc[2], acc[3]);
            const float2 r = __fadd2_rn(r01, r23);
            l_run = l_run * alpha + (r.x + r.y);
          } else {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const float2 x = make_float2(__uint_as_float(s[2 * i]), __uint_as_float(s[2 * i + 1]));
              float p0, p1;
              // BIAS: s already holds the biased logit (SiLU: its half)
              const float sm = BIAS ? 1.f : a.scale;
              if constexpr (PHI == GDPA_PHI_SILU) {
                // x * logistic(x) = x/2 * (1 + tanh(x/2)), x = s * scale
                const float2 hx =
                    BIAS ? x : __fmul2_rn(x, make_float2(half_scale, half_scale));
                const float2 t = make_float2(tanh_approx(hx.x), tanh_approx(hx.y));
                const float2 y = __ffma2_rn(hx, t, hx);
                p0 = y.x;
                p1 = y.y;
              } else if constexpr (PHI == GDPA_PHI_RELU) {
                p0 = relu_f(x.x * sm);
                p1 = relu_f(x.y * sm);
              } else if constexpr (PHI == GDPA_PHI_GELU) {
                const float2 y = gelu_f2(BIAS ? x : __fmul2_rn(x, make_float2(sm, sm)));
                p0 = y.x;
                p1 = y.y;
              } else {
                const float2 y = __fmul2_rn(x, make_float2(sm, sm));
                p0 = y.x;
                p1 = y.y;
              }
              pk[i] = pack_bf16x2(p0, p1);
            }
          }
        }
        // P_x is rewritten only once the previous PV_x has read it
        if (sc > 0) {
          w = mbar_wait(bar(C::B_PFREE + grp), (sc - 1) & 1u, abort_flag, kTimeoutNs);
          if (!__all_sync(0xffffffffu, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        {
          if (SOFTMAX && __any_sync(0xffffffffu, resc)) {
#pragma unroll
            for (int c = 0; c < DH; c += 16) {
              uint32_t ov[16];
              tmem_ld_x16(my_o + c, ov);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
              tmem_st_x16(my_o + c, ov);
            }
          }
          tmem_st_x32(my_p, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
          tmem_st_x32(my_p + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar(C::B_PFULL + grp));
      }
      if (!ok) break;
      // ---------------------------------------------------------- epilogue
      bool w = mbar_wait(bar(C::B_OFULL + grp), oc & 1u, abort_flag, kTimeoutNs);
      if (!__all_sync(0xffffffffu, w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      ++oc;
      const float inv = SOFTMAX ? 1.f / l_run : 1.f;
      // GDPA: rows of the tile in o [T, h, DH]; pooling: the seeds of (b, head) in o [B, h, S, DH]
      __nv_bfloat16* obase = POOL ? a.o + ((int64_t)tl.b * a.h + tl.head) * a.S * DH
                                  : a.o + ((int64_t)tl.row0 * a.h + tl.head) * DH;
      store_o_rows<DH>(my_o, base + C::OFF_OSTG + (uint32_t)(warp - 4) * C::OSTG_WARP, inv,
                       out_rows, quad, lane, obase, POOL ? (int64_t)DH : (int64_t)a.h * DH,
                       bar(C::B_OEMPTY + grp),
                       BIAS && a.b2 ? a.b2 + ((int64_t)tl.b * a.h + tl.head) * DH : nullptr);
      if (SOFTMAX && row < out_rows && a.lse != nullptr) {
        const int64_t at = POOL ? ((int64_t)tl.b * a.h + tl.head) * a.S + row
                                : (int64_t)tl.head * a.T + tl.row0 + row;
        a.lse[at] = (m_run + __log2f(l_run)) * 0.69314718055994531f;
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncwarp();
  __syncthreads();
  if (*abort_flag) {
    report(a.ws, GDPA_ERR_TIMEOUT);
    volatile int never = 0;
    if ((warp == 1 || warp == 3) && lane == 0) {         // both issuers' MMAs
      mma_commit(bar(C::B_DRAIN));
      mbar_wait(bar(C::B_DRAIN), 0, &never, kTimeoutNs);
    }
    if (warp == 0 && lane == 0) {                         // let in-flight TMA loads land
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
bool make_maps(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
               CUtensorMap* mq, CUtensorMap* mk, CUtensorMap* mv) {
  using C = FwdCfg<DH>;
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  const CUtensorMapSwizzle sw = DH < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  {
    const cuuint64_t dims[3] = {(cuuint64_t)DH, (cuuint64_t)p.h, (cuuint64_t)p.total_tokens};
    const cuuint64_t strides[2] = {(cuuint64_t)DH * 2, (cuuint64_t)p.h * DH * 2};
    const cuuint32_t box[3] = {(cuuint32_t)C::CH, 1, 128};
    if (enc(mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  const cuuint64_t dims[4] = {(cuuint64_t)DH, (cuuint64_t)p.m, (cuuint64_t)p.h, (cuuint64_t)p.B};
  const cuuint64_t strides[3] = {(cuuint64_t)DH * 2, (cuuint64_t)p.m * DH * 2,
                                 (cuuint64_t)p.h * p.m * DH * 2};
  const cuuint32_t box[4] = {(cuuint32_t)C::CH, 128, 1, 1};
  for (int i = 0; i < 2; ++i) {
    if (enc(i ? mv : mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(i ? v : k), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  return true;
}

// dh <= 64 (P in TMEM columns of its own): S released early; dh = 128: P aliases S.
template <int DH, int PHI, bool BIAS, bool KEYMASK>
constexpr auto fwd_kernel() {
  if constexpr (DH <= 64)
    return gdpa_fwd_early_kernel<DH, PHI, BIAS, kModeGdpa, KEYMASK>;
  else
    return gdpa_fwd_sm100_kernel<DH, PHI, BIAS, KEYMASK>;
}

template <int DH, int PHI, bool BIAS>
cudaError_t launch_fwd_t(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
                         const Bias& bs, void* o, float* lse, WsHeader* ws, const Tile* tiles,
                         cudaStream_t st) {
  using C = FwdCfg<DH>;
  CUtensorMap mq, mk, mv;
  if (!make_maps<DH>(p, q, k, v, &mq, &mk, &mv)) return cudaErrorInvalidValue;
  // softmax over a last key block with fewer than 128 keys needs the key mask
  // (the other activations give 0 on the zero-filled keys past m)
  auto kern = PHI == GDPA_PHI_SOFTMAX && p.m % 128 != 0 ? fwd_kernel<DH, PHI, BIAS, true>()
                                                         : fwd_kernel<DH, PHI, BIAS, false>();
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  FwdArgs args = {};
  args.tiles = tiles;
  args.ws = ws;
  args.o = reinterpret_cast<__nv_bfloat16*>(o);
  args.lse = lse;
  args.b1 = bs.b1;
  args.b2 = bs.b2;
  args.T = p.total_tokens;
  args.h = p.h;
  args.m = p.m;
  args.nkv = (p.m + 127) / 128;
  args.scale = p.scale;
  args.scale_log2 = p.scale * 1.4426950408889634f;
  KernelScope ks_("gdpa_fwd_sm100", st);
  kern<<<device_sm_count(), kThreads, C::SMEM, st>>>(mq, mk, mv, args);
  return cudaGetLastError();
}

template <int DH, bool BIAS>
cudaError_t launch_fwd_dh(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
                          const Bias& bs, void* o, float* lse, WsHeader* ws, const Tile* tiles,
                          cudaStream_t st) {
#define GDPA_FWD_PHI(PHIV) launch_fwd_t<DH, PHIV, BIAS>(p, q, k, v, bs, o, lse, ws, tiles, st)
  switch (p.phi) {
    case GDPA_PHI_SOFTMAX: return GDPA_FWD_PHI(GDPA_PHI_SOFTMAX);
    case GDPA_PHI_SILU: return GDPA_FWD_PHI(GDPA_PHI_SILU);
    case GDPA_PHI_RELU: return GDPA_FWD_PHI(GDPA_PHI_RELU);
    case GDPA_PHI_GELU: return GDPA_FWD_PHI(GDPA_PHI_GELU);
    default: return GDPA_FWD_PHI(GDPA_PHI_IDENTITY);
  }
#undef GDPA_FWD_PHI
}

template <int DH>
cudaError_t launch_fwd_bias(const gdpa_problem_t& p, const void* q, const void* k,
                            const void* v, const Bias& bs, void* o, float* lse, WsHeader* ws,
                            const Tile* tiles, cudaStream_t st) {
  if (bs.b1 || bs.b2) return launch_fwd_dh<DH, true>(p, q, k, v, bs, o, lse, ws, tiles, st);
  return launch_fwd_dh<DH, false>(p, q, k, v, bs, o, lse, ws, tiles, st);
}

// Sliding-window self-attention on the dh <= 64 forward kernel: q, k, v all
// jagged [T, h, DH] (one 3-D map each), work items = query tiles x head pairs.
template <int DH>
cudaError_t launch_window_t(int h, int64_t T, int window, float scale, const int32_t* offsets,
                            const void* q, const void* k, const void* v, void* o, float* lse,
                            WsHeader* ws, const Tile* tiles, cudaStream_t st) {
  using C = FwdCfg<DH>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorInvalidValue;
  const CUtensorMapSwizzle sw = DH < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint32_t estr[3] = {1, 1, 1};
  const cuuint64_t dims[3] = {(cuuint64_t)DH, (cuuint64_t)h, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)DH * 2, (cuuint64_t)h * DH * 2};
  const cuuint32_t box[3] = {(cuuint32_t)C::CH, 1, 128};
  CUtensorMap maps[3];
  const void* ptrs[3] = {q, k, v};
  for (int i = 0; i < 3; ++i)
    if (enc(&maps[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptrs[i]), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  auto kern = gdpa_fwd_early_kernel<DH, GDPA_PHI_SOFTMAX, false, kModeWindow>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  FwdArgs args = {};
  args.tiles = tiles;
  args.ws = ws;
  args.o = reinterpret_cast<__nv_bfloat16*>(o);
  args.lse = lse;
  args.T = T;
  args.h = h;
  args.window = window;
  args.offsets = offsets;
  args.scale = scale;
  args.scale_log2 = scale * 1.4426950408889634f;
  KernelScope ks_("gdpa_window_fwd_sm100", st);
  kern<<<device_sm_count(), kThreads, C::SMEM, st>>>(maps[0], maps[1], maps[2], args);
  return cudaGetLastError();
}

// Seed-query pooling on the dh <= 64 forward kernel: seeds [h, S, DH] as the
// query tiles (rows >= S read as zero), the jagged tokens [T, h, DH] as keys
// and values, softmax over each sample's tokens.
template <int DH>
cudaError_t launch_pool_t(int B, int h, int S, int64_t T, float scale, const void* seeds,
                          const void* k, const void* v, void* o, float* lse, WsHeader* ws,
                          const Tile* tiles, cudaStream_t st) {
  using C = FwdCfg<DH>;
  auto enc = tensor_map_encoder();
  if (!enc) return cudaErrorInvalidValue;
  const CUtensorMapSwizzle sw = DH < 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  const cuuint32_t estr[3] = {1, 1, 1};
  CUtensorMap mq, mk, mv;
  {
    const cuuint64_t dims[3] = {(cuuint64_t)DH, (cuuint64_t)S, (cuuint64_t)h};
    const cuuint64_t strides[2] = {(cuuint64_t)DH * 2, (cuuint64_t)S * DH * 2};
    const cuuint32_t box[3] = {(cuuint32_t)C::CH, 128, 1};
    if (enc(&mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(seeds), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const cuuint64_t dims[3] = {(cuuint64_t)DH, (cuuint64_t)h, (cuuint64_t)T};
  const cuuint64_t strides[2] = {(cuuint64_t)DH * 2, (cuuint64_t)h * DH * 2};
  const cuuint32_t box[3] = {(cuuint32_t)C::CH, 1, 128};
  for (int i = 0; i < 2; ++i)
    if (enc(i ? &mv : &mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(i ? v : k), dims,
            strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  auto kern = gdpa_fwd_early_kernel<DH, GDPA_PHI_SOFTMAX, false, kModePool>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  FwdArgs args = {};
  args.tiles = tiles;
  args.ws = ws;
  args.o = reinterpret_cast<__nv_bfloat16*>(o);
  args.lse = lse;
  args.T = T;
  args.h = h;
  args.m = 0;
  args.nkv = 0;
  args.S = S;
  args.scale = scale;
  args.scale_log2 = scale * 1.4426950408889634f;
  KernelScope ks_("gdpa_pool_fwd_sm100", st);
  kern<<<device_sm_count(), kThreads, C::SMEM, st>>>(mq, mk, mv, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sm100_fwd(const gdpa_problem_t& p, const void* q, const void* k,
                             const void* v, const Bias& bs, void* o, float* lse, WsHeader* ws,
                             const Tile* tiles, cudaStream_t st) {
  if (p.total_tokens == 0) return cudaSuccess;
  switch (p.dh) {
    case 32: return launch_fwd_bias<32>(p, q, k, v, bs, o, lse, ws, tiles, st);
    case 64: return launch_fwd_bias<64>(p, q, k, v, bs, o, lse, ws, tiles, st);
    case 128: return launch_fwd_bias<128>(p, q, k, v, bs, o, lse, ws, tiles, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_sm100_pool(int B, int h, int dh, int S, int64_t T, float scale,
                              const void* seeds, const void* k, const void* v, void* o,
                              float* lse, WsHeader* ws, const Tile* tiles, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (dh == 32) return launch_pool_t<32>(B, h, S, T, scale, seeds, k, v, o, lse, ws, tiles, st);
  if (dh == 64) return launch_pool_t<64>(B, h, S, T, scale, seeds, k, v, o, lse, ws, tiles, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_sm100_window(int h, int dh, int64_t T, int window, float scale,
                                const int32_t* offsets, const void* q, const void* k,
                                const void* v, void* o, float* lse, WsHeader* ws,
                                const Tile* tiles, cudaStream_t st) {
  if (T == 0) return cudaSuccess;
  if (dh == 32)
    return launch_window_t<32>(h, T, window, scale, offsets, q, k, v, o, lse, ws, tiles, st);
  if (dh == 64)
    return launch_window_t<64>(h, T, window, scale, offsets, q, k, v, o, lse, ws, tiles, st);
  return cudaErrorInvalidValue;
}

}  // namespace gdpa
