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
  int64_t T;
  int h, m, nkv;
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
  // barrier slots
  static constexpr int B_QFULL = 0, B_QEMPTY = 2, B_SFULL = 4, B_PFULL = 6, B_OFULL = 8,
                       B_OEMPTY = 10, B_DRAIN = 12, B_KVFULL = 13, B_KVEMPTY = 13 + NS,
                       NBAR = 13 + 2 * NS;
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

template <int DH, int PHI>
__global__ void __launch_bounds__(kThreads, 1)
gdpa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const FwdArgs a) {
  using C = FwdCfg<DH>;
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
      for (int j = 0; j < nkv; ++j, ++sc) {
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
          };
          auto row_max = [&]() -> float {
            float m8[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) m8[u] = c2 >= 0.f ? -INFINITY : INFINITY;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              load_half(hf);
#pragma unroll
              for (int i = 0; i < 64; ++i) {
                const float x = __uint_as_float(sh[i]);
                if (valid == C::BN || 64 * hf + i < valid)
                  m8[i & 7] = c2 >= 0.f ? fmaxf(m8[i & 7], x) : fminf(m8[i & 7], x);
              }
            }
#pragma unroll
            for (int u = 4; u > 0; u >>= 1)
#pragma unroll
              for (int v = 0; v < u; ++v)
                m8[v] = c2 >= 0.f ? fmaxf(m8[v], m8[v + u]) : fminf(m8[v], m8[v + u]);
            return m8[0] * c2;
          };
          uint32_t pk[C::P_SEP ? 32 : 64];
          auto exp_pack = [&]() -> float {
            const float neg_m = -m_run;
            float rs8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              load_half(hf);
              uint32_t* pkh = C::P_SEP ? pk : pk + 32 * hf;
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int col = 64 * hf + 2 * i;
                float p0 = ex2_approx(fmaf(__uint_as_float(sh[2 * i]), c2, neg_m));
                float p1 = ex2_approx(fmaf(__uint_as_float(sh[2 * i + 1]), c2, neg_m));
                if (valid < C::BN) {
                  p0 = col < valid ? p0 : 0.f;
                  p1 = col + 1 < valid ? p1 : 0.f;
                }
                rs8[(2 * i) & 7] += p0;
                rs8[(2 * i + 1) & 7] += p1;
                pkh[i] = pack_bf16x2(p0, p1);
              }
              if (C::P_SEP) tmem_st_x32(my_p + 32 * hf, *reinterpret_cast<uint32_t(*)[32]>(pkh));
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
          if (!C::P_SEP) {
            tmem_st_x32(my_s + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
            tmem_st_x32(my_s + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
          }
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
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float x0 = __uint_as_float(s[2 * i]), x1 = __uint_as_float(s[2 * i + 1]);
              float p0, p1;
              if constexpr (PHI == GDPA_PHI_SILU) {
                p0 = silu_tanh(x0, half_scale);
                p1 = silu_tanh(x1, half_scale);
              } else if constexpr (PHI == GDPA_PHI_RELU) {
                p0 = relu_f(x0 * a.scale);
                p1 = relu_f(x1 * a.scale);
              } else if constexpr (PHI == GDPA_PHI_GELU) {
                p0 = gelu_f(x0 * a.scale);
                p1 = gelu_f(x1 * a.scale);
              } else {
                p0 = x0 * a.scale;
                p1 = x1 * a.scale;
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
      {
        // Each lane owns one O row.  The warp passes its 32 rows through
        // shared memory (64 columns at a time, rows swizzled by 16-byte
        // chunk) so that every global store instruction writes whole rows:
        // CPR lanes per row, 32 / CPR rows per instruction.
        constexpr int PC = DH < 64 ? DH : 64;           // columns per pass
        constexpr int CPR = PC / 8;                     // 16-byte chunks per row
        constexpr int RPI = 32 / CPR;                   // rows per store instruction
        const uint32_t ostg = base + C::OFF_OSTG + (uint32_t)(warp - 4) * C::OSTG_WARP;
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
            mbar_arrive(bar(C::B_OEMPTY + grp));        // the O accumulator is free
          }
#pragma unroll
          for (int j = 0; j < CPR; ++j) {
            const uint32_t p0 = pack_bf16x2(__uint_as_float(v[8 * j]) * inv, __uint_as_float(v[8 * j + 1]) * inv);
            const uint32_t p1 = pack_bf16x2(__uint_as_float(v[8 * j + 2]) * inv, __uint_as_float(v[8 * j + 3]) * inv);
            const uint32_t p2 = pack_bf16x2(__uint_as_float(v[8 * j + 4]) * inv, __uint_as_float(v[8 * j + 5]) * inv);
            const uint32_t p3 = pack_bf16x2(__uint_as_float(v[8 * j + 6]) * inv, __uint_as_float(v[8 * j + 7]) * inv);
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
            if (tr < tl.rows)
              *reinterpret_cast<uint4*>(a.o + ((int64_t)(tl.row0 + tr) * a.h + tl.head) * DH + c0 +
                                        jl * 8) = val;
          }
          __syncwarp();
        }
      }
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

template <int DH, int PHI>
cudaError_t launch_fwd_t(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
                         void* o, float* lse, WsHeader* ws, const Tile* tiles, cudaStream_t st) {
  using C = FwdCfg<DH>;
  CUtensorMap mq, mk, mv;
  if (!make_maps<DH>(p, q, k, v, &mq, &mk, &mv)) return cudaErrorInvalidValue;
  auto kern = gdpa_fwd_sm100_kernel<DH, PHI>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
  if (e != cudaSuccess) return e;
  FwdArgs args;
  args.tiles = tiles;
  args.ws = ws;
  args.o = reinterpret_cast<__nv_bfloat16*>(o);
  args.lse = lse;
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

template <int DH>
cudaError_t launch_fwd_dh(const gdpa_problem_t& p, const void* q, const void* k, const void* v,
                          void* o, float* lse, WsHeader* ws, const Tile* tiles, cudaStream_t st) {
  switch (p.phi) {
    case GDPA_PHI_SOFTMAX: return launch_fwd_t<DH, GDPA_PHI_SOFTMAX>(p, q, k, v, o, lse, ws, tiles, st);
    case GDPA_PHI_SILU: return launch_fwd_t<DH, GDPA_PHI_SILU>(p, q, k, v, o, lse, ws, tiles, st);
    case GDPA_PHI_RELU: return launch_fwd_t<DH, GDPA_PHI_RELU>(p, q, k, v, o, lse, ws, tiles, st);
    case GDPA_PHI_GELU: return launch_fwd_t<DH, GDPA_PHI_GELU>(p, q, k, v, o, lse, ws, tiles, st);
    default: return launch_fwd_t<DH, GDPA_PHI_IDENTITY>(p, q, k, v, o, lse, ws, tiles, st);
  }
}

}  // namespace

cudaError_t launch_sm100_fwd(const gdpa_problem_t& p, const void* q, const void* k,
                             const void* v, void* o, float* lse, WsHeader* ws, const Tile* tiles,
                             cudaStream_t st) {
  if (p.total_tokens == 0) return cudaSuccess;
  switch (p.dh) {
    case 32: return launch_fwd_dh<32>(p, q, k, v, o, lse, ws, tiles, st);
    case 64: return launch_fwd_dh<64>(p, q, k, v, o, lse, ws, tiles, st);
    case 128: return launch_fwd_dh<128>(p, q, k, v, o, lse, ws, tiles, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gdpa
