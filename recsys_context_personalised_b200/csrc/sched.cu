// Jagged tile scheduler: device offsets -> list of (sample, head, row range)
// work items, with no host synchronisation.
//
// Samples have different history lengths n_b (the Kunlun summary, section 1,
// names irregular tensor shapes as a cause of low utilisation).  Every sample
// b is cut into ceil(n_b / bm) query tiles; item order is sample-major, then
// head, then tile, so the tiles that share one (sample, head) key/value set
// are adjacent in the list and run at the same time on neighbouring SMs,
// which keeps that K/V set resident in L2.
#include "gdpa_internal.cuh"

namespace gdpa {

int device_sm_count();

namespace {

constexpr int kSchedThreads = 1024;
constexpr int kSortMax = 4096;   // samples whose per-sample data a CTA keeps in shared memory

// Checks the offsets (offsets[0] = 0, offsets[B] = T, 0 <= n_b <= max_n) in
// every CTA; CTA 0 records the outcome in the workspace header.  Returns
// whether they are valid (the same answer in every thread of the grid).
__device__ bool offsets_valid(const int32_t* __restrict__ offsets, int B, int64_t T, int max_n,
                              WsHeader* ws, int* s_bad) {
  const int tid = threadIdx.x;
  if (tid == 0) *s_bad = (offsets[0] != 0 || (int64_t)offsets[B] != T) ? 1 : 0;
  __syncthreads();
  for (int b = tid; b < B; b += blockDim.x) {
    const int n = offsets[b + 1] - offsets[b];
    if (n < 0 || n > max_n) *s_bad = 1;
  }
  __syncthreads();
  const bool ok = *s_bad == 0;
  if (blockIdx.x == 0 && tid == 0) {
    ws->status = ok ? GDPA_OK : GDPA_ERR_INVALID_ARG;
    if (!ok) ws->tile_count = 0;
  }
  return ok;
}

// Exclusive prefix sums of cnt(i), i in [0, N), handed to put(i, sum);
// returns the total.  All threads of the block take part; thread i reads
// cnt(i) before any put of its chunk.
template <typename F, typename G>
__device__ long long block_prefix(int N, F cnt, G put, int* s_warp, long long* s_carry) {
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
  if (tid == 0) *s_carry = 0;
  __syncthreads();
  for (int base = 0; base < N; base += blockDim.x) {
    const int i = base + tid;
    const int v = i < N ? cnt(i) : 0;
    int x = v;                                      // inclusive scan within the warp
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, d);
      if (lane >= d) x += y;
    }
    if (lane == 31) s_warp[wid] = x;
    __syncthreads();
    if (wid == 0) {                                 // scan of the warp totals
      int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, w, d);
        if (lane >= d) w += y;
      }
      if (lane < nw) s_warp[lane] = w;             // inclusive
    }
    __syncthreads();
    const long long before = *s_carry + (wid > 0 ? s_warp[wid - 1] : 0);
    if (i < N) put(i, (int)(before + x - v));
    __syncthreads();
    if (tid == 0) *s_carry += s_warp[nw - 1];
    __syncthreads();
  }
  return *s_carry;
}

// The largest i in [0, N) with h * pre(i) <= idx (pre non-decreasing, pre(0) = 0).
template <typename F>
__device__ __forceinline__ int find_owner(F pre, int N, int h, long long idx) {
  int lo = 0, hi = N - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((long long)h * pre(mid) <= idx) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kSchedThreads)
schedule_kernel(const int32_t* __restrict__ offsets, int B, int h, int64_t T, int max_n,
                int bm, WsHeader* ws, Tile* __restrict__ tiles, int64_t cap) {
  __shared__ int s_bad;
  __shared__ int s_pre[kSortMax];
  __shared__ int s_warp[32];
  __shared__ long long s_carry;
  if (!offsets_valid(offsets, B, T, max_n, ws, &s_bad)) return;
  const int tid = threadIdx.x;
  if (B <= kSortMax) {
    // every CTA forms the prefix of the tile counts, then the grid writes the
    // items, each thread finding its item's sample by binary search
    auto ntiles = [&](int b) { return (offsets[b + 1] - offsets[b] + bm - 1) / bm; };
    auto put = [&](int b, int v) { s_pre[b] = v; };
    auto pre = [&](int b) { return s_pre[b]; };
    const long long total = block_prefix(B, ntiles, put, s_warp, &s_carry);
    const long long items = (long long)h * total < cap ? (long long)h * total : cap;
    for (long long idx = (long long)blockIdx.x * blockDim.x + tid; idx < items;
         idx += (long long)gridDim.x * blockDim.x) {
      const int b = find_owner(pre, B, h, idx);
      const int n = offsets[b + 1] - offsets[b];
      const int nt = (n + bm - 1) / bm;
      const int rem = (int)(idx - (long long)h * s_pre[b]);
      const int t = rem % nt;
      Tile w;
      w.b = b;
      w.head = rem / nt;
      w.row0 = offsets[b] + t * bm;
      w.rows = min(bm, n - t * bm);
      tiles[idx] = w;
    }
    if (blockIdx.x == 0 && tid == 0) ws->tile_count = (int)items;
    return;
  }
  // more samples than a CTA keeps: CTA 0 alone, one thread per sample
  if (blockIdx.x != 0) return;
  int* s_scan = s_pre;
  if (tid == 0) s_carry = 0;
  __syncthreads();
  for (int base = 0; base < B; base += kSchedThreads) {
    const int b = base + tid;
    const int n = b < B ? offsets[b + 1] - offsets[b] : 0;
    const int nt = (n + bm - 1) / bm;
    s_scan[tid] = nt;
    __syncthreads();
    for (int d = 1; d < kSchedThreads; d <<= 1) {
      const int add = tid >= d ? s_scan[tid - d] : 0;
      __syncthreads();
      s_scan[tid] += add;
      __syncthreads();
    }
    const long long excl = s_carry + s_scan[tid] - nt;
    if (b < B) {
      const int t0 = offsets[b];
      for (int j = 0; j < h; ++j)
        for (int t = 0; t < nt; ++t) {
          const long long idx = (long long)h * excl + (long long)j * nt + t;
          if (idx < cap) {
            Tile w;
            w.b = b;
            w.head = j;
            w.row0 = t0 + t * bm;
            w.rows = min(bm, n - t * bm);
            tiles[idx] = w;
          }
        }
    }
    __syncthreads();
    if (tid == kSchedThreads - 1) s_carry += s_scan[kSchedThreads - 1];
    __syncthreads();
  }
  if (tid == 0) {
    const long long total = (long long)h * s_carry;
    ws->tile_count = (int)(total < cap ? total : cap);
  }
}

// Sorts the samples by length, longest first (ties: lower index first), into
// s_key[0, B) as (n_b, b); entries [B, P2) pad with (-1, INT_MAX).  B <= kSortMax.
// A bitonic sorting network over the next power of two P2, all threads taking
// part (Batcher, "Sorting networks and their applications", AFIPS 1968).
__device__ void sort_by_length(const int32_t* __restrict__ offsets, int B, int2* s_key) {
  const int tid = threadIdx.x;
  int P2 = 1;
  while (P2 < B) P2 <<= 1;
  for (int i = tid; i < P2; i += kSchedThreads)
    s_key[i] = i < B ? make_int2(offsets[i + 1] - offsets[i], i) : make_int2(-1, 0x7fffffff);
  __syncthreads();
  for (int k = 2; k <= P2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P2; i += kSchedThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const int2 x = s_key[i], y = s_key[ixj];
          const bool x_first = x.x > y.x || (x.x == y.x && x.y < y.y);
          const bool up = (i & k) == 0;
          if (up ? !x_first : x_first) {
            s_key[i] = y;
            s_key[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// Backward work list: one item per (sample, head, 128-key block), samples in
// decreasing length order (longest-processing-time first), so that a static
// round-robin over CTAs gives every SM about the same number of query tiles.
// Item fields: b, head, row0 = first key of the block, rows = n_b.

__global__ void __launch_bounds__(kSchedThreads)
schedule_kv_kernel(const int32_t* __restrict__ offsets, int B, int h, int64_t T, int max_n,
                   int nkv, WsHeader* ws, Tile* __restrict__ tiles) {
  __shared__ int s_bad;
  __shared__ int2 s_key[kSortMax];   // (n_b, b)
  if (!offsets_valid(offsets, B, T, max_n, ws, &s_bad)) return;
  // every CTA sorts; the grid writes the items
  const bool sorted = B <= kSortMax;
  if (sorted) sort_by_length(offsets, B, s_key);
  const long long per_sample = (long long)h * nkv;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
       idx < (long long)B * per_sample; idx += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(idx / per_sample);
    const int rem = (int)(idx % per_sample);
    const int b = sorted ? s_key[r].y : r;
    Tile w;
    w.b = b;
    w.head = rem / nkv;
    w.row0 = (rem % nkv) * 128;
    w.rows = offsets[b + 1] - offsets[b];
    tiles[idx] = w;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) ws->tile_count = (int)((long long)B * per_sample);
}

// Seed-pooling work list: one item per (sample, pair of heads 2k, 2k+1) of the
// samples that have tokens, longest samples first (B <= 4096): item fields
// b, head = 2k, row0 = offsets[b], rows = n_b.  Samples without tokens get no
// item (pool_empty_kernel writes their outputs).
__global__ void __launch_bounds__(kSchedThreads)
schedule_pool_kernel(const int32_t* __restrict__ offsets, int B, int h, int64_t T, int max_n,
                     WsHeader* ws, Tile* __restrict__ tiles) {
  __shared__ int s_bad;
  __shared__ int s_nz;
  __shared__ int2 s_key[kSortMax];   // (n_b, b)
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_bad = 0;
    s_nz = 0;
    ws->status = GDPA_OK;
    if (offsets[0] != 0 || (int64_t)offsets[B] != T) s_bad = 1;
  }
  __syncthreads();
  for (int b = tid; b < B; b += kSchedThreads) {
    const int n = offsets[b + 1] - offsets[b];
    if (n < 0 || n > max_n) s_bad = 1;
    if (n > 0) atomicAdd(&s_nz, 1);
  }
  __syncthreads();
  if (s_bad) {
    if (tid == 0) {
      ws->status = GDPA_ERR_INVALID_ARG;
      ws->tile_count = 0;
    }
    return;
  }
  sort_by_length(offsets, B, s_key);         // samples without tokens sort last
  const int hp = (h + 1) / 2;
  const long long items = (long long)s_nz * hp;
  for (long long idx = tid; idx < items; idx += kSchedThreads) {
    const int b = s_key[(int)(idx / hp)].y;
    Tile w;
    w.b = b;
    w.head = 2 * (int)(idx % hp);
    w.row0 = offsets[b];
    w.rows = offsets[b + 1] - offsets[b];
    tiles[idx] = w;
  }
  if (tid == 0) ws->tile_count = (int)items;
}

// Backward work list of the variants whose keys are the jagged tokens (seed
// pooling, the sliding window): one item per (sample, head, 128-token key
// block) of the samples that have tokens, samples in decreasing length order
// (B <= 4096), head-major within a sample.  Item fields: b, head, row0 = first
// key of the block (sample-local), rows = n_b.
__global__ void __launch_bounds__(kSchedThreads)
schedule_jkv_kernel(const int32_t* __restrict__ offsets, int B, int h, int64_t T, int max_n,
                    WsHeader* ws, Tile* __restrict__ tiles, int64_t cap) {
  __shared__ int s_bad;
  __shared__ int s_warp[32];
  __shared__ long long s_carry;
  __shared__ int2 s_key[kSortMax];   // (n_b, b), then (prefix of the key-block counts, b)
  if (!offsets_valid(offsets, B, T, max_n, ws, &s_bad)) return;
  // every CTA sorts and forms the prefix of the key-block counts in sorted
  // order (samples without tokens sort last); the grid writes the items
  sort_by_length(offsets, B, s_key);
  auto nblocks = [&](int r) { return (max(s_key[r].x, 0) + 127) >> 7; };
  auto put = [&](int r, int v) { s_key[r].x = v; };
  auto pre = [&](int r) { return s_key[r].x; };
  const long long total = block_prefix(B, nblocks, put, s_warp, &s_carry);
  const long long items = (long long)h * total < cap ? (long long)h * total : cap;
  for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < items;
       idx += (long long)gridDim.x * blockDim.x) {
    const int r = find_owner(pre, B, h, idx);
    const int b = s_key[r].y;
    const int n = offsets[b + 1] - offsets[b];
    const int nb = (n + 127) >> 7;
    const int rem = (int)(idx - (long long)h * s_key[r].x);
    Tile w;
    w.b = b;
    w.head = rem / nb;
    w.row0 = 128 * (rem % nb);
    w.rows = n;
    tiles[idx] = w;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) ws->tile_count = (int)items;
}

// Outputs of the samples without tokens: O = 0 and LSE = -inf (every seed
// pools over an empty set).  One thread per 8 columns of an output row.
__global__ void pool_empty_kernel(const int32_t* __restrict__ offsets, int B, int h, int S,
                                  int dh, uint4* __restrict__ o, float* __restrict__ lse,
                                  const WsHeader* __restrict__ ws) {
  if (ws->status == GDPA_ERR_INVALID_ARG) return;
  const int per_row = dh / 8;
  const int64_t n = (int64_t)B * h * S * per_row;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int64_t row = i / per_row;                  // (b, head, seed)
    const int b = (int)(row / ((int64_t)h * S));
    if (offsets[b + 1] != offsets[b]) continue;
    o[i] = make_uint4(0u, 0u, 0u, 0u);
    if (lse != nullptr && i % per_row == 0) lse[row] = -INFINITY;
  }
}
}  // namespace

cudaError_t launch_schedule_kv(const gdpa_problem_t& p, const int32_t* offsets, WsHeader* ws,
                               Tile* tiles, cudaStream_t st) {
  KernelScope ks_("gdpa_schedule_kv", st);
  schedule_kv_kernel<<<device_sm_count(), kSchedThreads, 0, st>>>(offsets, p.B, p.h, p.total_tokens, p.max_n,
                                                   (p.m + 127) / 128, ws, tiles);
  return cudaGetLastError();
}

cudaError_t launch_schedule(const gdpa_problem_t& p, const int32_t* offsets, int bm,
                            WsHeader* ws, Tile* tiles, cudaStream_t st) {
  KernelScope ks_("gdpa_schedule", st);
  schedule_kernel<<<device_sm_count(), kSchedThreads, 0, st>>>(offsets, p.B, p.h, p.total_tokens, p.max_n,
                                                bm, ws, tiles, tile_capacity(p, bm));
  return cudaGetLastError();
}

}  // namespace gdpa

namespace gdpa {

cudaError_t launch_schedule_pool(const int32_t* offsets, int B, int h, int64_t T, int max_n,
                                 WsHeader* ws, Tile* tiles, cudaStream_t st) {
  KernelScope ks_("gdpa_schedule_pool", st);
  schedule_pool_kernel<<<1, kSchedThreads, 0, st>>>(offsets, B, h, T, max_n, ws, tiles);
  return cudaGetLastError();
}

cudaError_t launch_schedule_jkv(const int32_t* offsets, int B, int h, int64_t T, int max_n,
                                WsHeader* ws, Tile* tiles, int64_t cap, cudaStream_t st) {
  KernelScope ks_("gdpa_schedule_jkv", st);
  schedule_jkv_kernel<<<device_sm_count(), kSchedThreads, 0, st>>>(offsets, B, h, T, max_n, ws, tiles, cap);
  return cudaGetLastError();
}

cudaError_t launch_pool_empty(const int32_t* offsets, int B, int h, int S, int dh, void* o,
                              float* lse, const WsHeader* ws, cudaStream_t st) {
  const int64_t n = (int64_t)B * h * S * (dh / 8);
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  KernelScope ks_("gdpa_pool_empty", st);
  pool_empty_kernel<<<(unsigned)blocks, 256, 0, st>>>(offsets, B, h, S, dh, (uint4*)o, lse, ws);
  return cudaGetLastError();
}

}  // namespace gdpa
