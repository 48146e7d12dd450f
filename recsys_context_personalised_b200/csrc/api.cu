// C ABI entry points of libgdpa.so: argument validation, workspace layout and
// kernel dispatch.  Every step of the operator runs in this library's kernels.
#include <stdio.h>
#include <string.h>

#include <string>
#include <vector>

#include "gdpa_internal.cuh"

namespace gdpa {

static thread_local int g_launches = 0;

struct TimingRec {
  const char* name;
  cudaEvent_t start, stop;
};
static thread_local bool g_timing = false;
static thread_local std::vector<TimingRec> g_recs;

KernelScope::KernelScope(const char* name, cudaStream_t s) : rec(-1), st(s) {
  ++g_launches;
  if (!g_timing) return;
  TimingRec r{name, nullptr, nullptr};
  if (cudaEventCreate(&r.start) != cudaSuccess || cudaEventCreate(&r.stop) != cudaSuccess) return;
  cudaEventRecord(r.start, st);
  g_recs.push_back(r);
  rec = (int)g_recs.size() - 1;
}

KernelScope::~KernelScope() {
  if (rec >= 0) cudaEventRecord(g_recs[rec].stop, st);
}

static void clear_records() {
  for (auto& r : g_recs) {
    if (r.start) cudaEventDestroy(r.start);
    if (r.stop) cudaEventDestroy(r.stop);
  }
  g_recs.clear();
}

// bf16 problems run on the tcgen05 kernels.
cudaError_t launch_sm100_fwd(const gdpa_problem_t& p, const void* q, const void* k,
                             const void* v, const Bias& bs, void* o, float* lse, WsHeader* ws,
                             const Tile* tiles, cudaStream_t st);
cudaError_t launch_sm100_bwd(const gdpa_problem_t& p, const void* q, const int32_t* offsets,
                             const void* k, const void* v, const Bias& bs, const void* o,
                             const float* lse, const void* dout, void* dq, void* dk, void* dv,
                             float* dq_acc, float* dsum, WsHeader* ws, Tile* tiles,
                             cudaStream_t st);
int64_t sm100_bwd_items(const gdpa_problem_t& p);
cudaError_t launch_sm100_window(int h, int dh, int64_t T, int window, float scale,
                                const int32_t* offsets, const void* q, const void* k,
                                const void* v, void* o, float* lse, WsHeader* ws,
                                const Tile* tiles, cudaStream_t st);
cudaError_t launch_sm100_pool(int B, int h, int dh, int S, int64_t T, float scale,
                              const void* seeds, const void* k, const void* v, void* o,
                              float* lse, WsHeader* ws, const Tile* tiles, cudaStream_t st);
cudaError_t launch_sm100_window_bwd(int B, int h, int dh, int64_t T, int max_n, int window,
                                    float scale, const int32_t* offsets, const void* q,
                                    const void* k, const void* v, const void* o,
                                    const float* lse, const void* dout, void* dq, void* dk,
                                    void* dv, float* dq_acc, float* dsum, WsHeader* ws,
                                    Tile* tiles, int64_t cap, cudaStream_t st);
cudaError_t launch_sm100_pool_bwd(int B, int h, int dh, int S, int64_t T, int max_n, float scale,
                                  const int32_t* offsets, const void* seeds, const void* k,
                                  const void* v, const void* o, const float* lse,
                                  const void* dout, float* dseeds, void* dk, void* dv,
                                  float* dsum, WsHeader* ws, Tile* tiles, int64_t cap,
                                  cudaStream_t st);

namespace {

struct FwdLayout {
  size_t tiles_off, total;
  int bm;
};
struct BwdLayout {
  size_t tiles_off, dsum_off, dqacc_off, total;
  int bm;
};

bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

gdpa_status_t check_problem(const gdpa_problem_t* p) {
  if (!p) return GDPA_ERR_INVALID_ARG;
  if (p->B < 1 || p->h < 1 || p->m < 1 || p->max_n < 0 || p->total_tokens < 0 ||
      p->total_tokens >= (int64_t)1 << 31)
    return GDPA_ERR_INVALID_ARG;
  if ((int64_t)p->max_n * p->B < p->total_tokens) return GDPA_ERR_INVALID_ARG;
  if (p->phi < GDPA_PHI_IDENTITY || p->phi > GDPA_PHI_GELU) return GDPA_ERR_INVALID_ARG;
  if (p->dtype != GDPA_DTYPE_F32 && p->dtype != GDPA_DTYPE_BF16) return GDPA_ERR_INVALID_ARG;
  if (!(p->scale == p->scale) || p->scale > 3.0e38f || p->scale < -3.0e38f)
    return GDPA_ERR_INVALID_ARG;
  if (p->dh != 32 && p->dh != 64 && p->dh != 128) return GDPA_ERR_UNSUPPORTED;
  // element counts must fit the kernels' 64-bit index math; K/V rows < 2^31
  if ((int64_t)p->B * p->h * p->m >= (int64_t)1 << 31) return GDPA_ERR_UNSUPPORTED;
  if ((int64_t)p->B * p->h >= (int64_t)1 << 24) return GDPA_ERR_UNSUPPORTED;
  return GDPA_OK;
}

// One backend per element type: bf16 runs on the tcgen05 kernels (128-row
// tiles), fp32 on the exact SIMT kernels (64-row tiles).
int fwd_bm(const gdpa_problem_t& p) { return p.dtype == GDPA_DTYPE_BF16 ? kMmaBM : kSimtBM; }
int bwd_bm(const gdpa_problem_t& p) { return p.dtype == GDPA_DTYPE_BF16 ? kMmaBM : kSimtBM; }

FwdLayout fwd_layout(const gdpa_problem_t& p) {
  FwdLayout L;
  L.bm = fwd_bm(p);
  L.tiles_off = sizeof(WsHeader);
  L.total = align_up(L.tiles_off + sizeof(Tile) * (size_t)tile_capacity(p, L.bm), 256);
  return L;
}

BwdLayout bwd_layout(const gdpa_problem_t& p) {
  BwdLayout L;
  L.bm = bwd_bm(p);
  L.tiles_off = sizeof(WsHeader);
  int64_t items = tile_capacity(p, L.bm);
  if (L.bm == kMmaBM) items = sm100_bwd_items(p);   // (sample, head, key block) list
  L.dsum_off = align_up(L.tiles_off + sizeof(Tile) * (size_t)items, 256);
  L.dqacc_off = align_up(L.dsum_off + sizeof(float) * (size_t)p.h * (size_t)p.total_tokens, 256);
  size_t dq_bytes = 0;
  if (L.bm == kMmaBM) dq_bytes = sizeof(float) * (size_t)p.total_tokens * p.h * p.dh;
  L.total = align_up(L.dqacc_off + dq_bytes, 256);
  return L;
}

gdpa_status_t check_ws(const void* ws, size_t have, size_t need) {
  if (!ws || ((uintptr_t)ws & 255u) != 0 || have < need) return GDPA_ERR_WORKSPACE;
  return GDPA_OK;
}

gdpa_status_t cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return GDPA_OK;
  fprintf(stderr, "gdpa: CUDA error %d (%s)\n", (int)e, cudaGetErrorString(e));
  return GDPA_ERR_CUDA;
}

}  // namespace
}  // namespace gdpa

using namespace gdpa;

extern "C" {

gdpa_status_t gdpa_fwd_workspace_size(const gdpa_problem_t* p, size_t* bytes) {
  gdpa_status_t s = check_problem(p);
  if (s != GDPA_OK) return s;
  if (!bytes) return GDPA_ERR_INVALID_ARG;
  *bytes = fwd_layout(*p).total;
  return GDPA_OK;
}

gdpa_status_t gdpa_bwd_workspace_size(const gdpa_problem_t* p, size_t* bytes) {
  gdpa_status_t s = check_problem(p);
  if (s != GDPA_OK) return s;
  if (!bytes) return GDPA_ERR_INVALID_ARG;
  *bytes = bwd_layout(*p).total;
  return GDPA_OK;
}

gdpa_status_t gdpa_fwd_bias(const gdpa_problem_t* p, const void* q, const int32_t* offsets,
                            const void* k, const void* v, const float* b1, const float* b2,
                            void* o, float* lse, void* workspace, size_t workspace_bytes,
                            void* stream) {
  g_launches = 0;
  gdpa_status_t s = check_problem(p);
  if (s != GDPA_OK) return s;
  // with no tokens there is nothing to read from q or write to o
  const bool empty = p->total_tokens == 0;
  if (!offsets || !k || !v || (!empty && (!q || !o))) return GDPA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      ((uintptr_t)offsets & 3u) || ((uintptr_t)lse & 3u) || ((uintptr_t)b1 & 3u) ||
      ((uintptr_t)b2 & 3u))
    return GDPA_ERR_INVALID_ARG;
  const FwdLayout L = fwd_layout(*p);
  s = check_ws(workspace, workspace_bytes, L.total);
  if (s != GDPA_OK) return s;
  if (p->phi != GDPA_PHI_SOFTMAX) lse = nullptr;
  Bias bs;
  bs.b1 = b1;
  bs.b2 = b2;
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* ws = (WsHeader*)workspace;
  Tile* tiles = (Tile*)((char*)workspace + L.tiles_off);
  cudaError_t e = launch_schedule(*p, offsets, L.bm, ws, tiles, st);
  if (e != cudaSuccess) return cuda_status(e);
  if (L.bm == kMmaBM)
    e = launch_sm100_fwd(*p, q, k, v, bs, o, lse, ws, tiles, st);
  else
    e = launch_simt_fwd(*p, q, k, v, bs, o, lse, ws, tiles, tile_capacity(*p, L.bm), st);
  return cuda_status(e);
}

gdpa_status_t gdpa_fwd(const gdpa_problem_t* p, const void* q, const int32_t* offsets,
                       const void* k, const void* v, void* o, float* lse, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return gdpa_fwd_bias(p, q, offsets, k, v, nullptr, nullptr, o, lse, workspace,
                       workspace_bytes, stream);
}

gdpa_status_t gdpa_bwd_bias(const gdpa_problem_t* p, const void* q, const int32_t* offsets,
                            const void* k, const void* v, const float* b1, const float* b2,
                            const void* o, const float* lse, const void* dout, void* dq,
                            void* dk, void* dv, float* db1, float* db2, void* workspace,
                            size_t workspace_bytes, void* stream) {
  g_launches = 0;
  gdpa_status_t s = check_problem(p);
  if (s != GDPA_OK) return s;
  // with no tokens q, o, lse, dout and dq are never touched; dk and dv are zeroed
  const bool empty = p->total_tokens == 0;
  if (!offsets || !k || !v || !dk || !dv) return GDPA_ERR_INVALID_ARG;
  if (!empty && (!q || !dout || !dq)) return GDPA_ERR_INVALID_ARG;
  if (!empty && p->phi == GDPA_PHI_SOFTMAX && (!o || !lse)) return GDPA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(dout) || !aligned16(dq) ||
      !aligned16(dk) || !aligned16(dv) || (o && !aligned16(o)) || ((uintptr_t)offsets & 3u) ||
      ((uintptr_t)lse & 3u) || ((uintptr_t)b1 & 3u) || ((uintptr_t)b2 & 3u) ||
      ((uintptr_t)db1 & 3u) || ((uintptr_t)db2 & 3u))
    return GDPA_ERR_INVALID_ARG;
  const BwdLayout L = bwd_layout(*p);
  s = check_ws(workspace, workspace_bytes, L.total);
  if (s != GDPA_OK) return s;
  Bias bs;
  bs.b1 = b1;
  bs.b2 = b2;
  bs.db1 = db1;
  bs.db2 = db2;
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* ws = (WsHeader*)workspace;
  Tile* tiles = (Tile*)((char*)workspace + L.tiles_off);
  float* dsum = (float*)((char*)workspace + L.dsum_off);
  if (L.bm == kMmaBM) {
    float* dq_acc = (float*)((char*)workspace + L.dqacc_off);
    return cuda_status(launch_sm100_bwd(*p, q, offsets, k, v, bs, o, lse, dout, dq, dk, dv,
                                        dq_acc, dsum, ws, tiles, st));
  }
  cudaError_t e = launch_schedule(*p, offsets, L.bm, ws, tiles, st);
  if (e != cudaSuccess) return cuda_status(e);
  const bool softmax = p->phi == GDPA_PHI_SOFTMAX;
  if (softmax && !b2) {
    e = launch_row_dot(*p, o, dout, dsum, st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  // db2, db1 = 0, and (with an output bias) the softmax row sums of O - b2
  e = launch_bias_prep(*p, offsets, o, dout, b2, softmax && b2 ? dsum : nullptr, db1, db2, ws,
                       st);
  if (e != cudaSuccess) return cuda_status(e);
  e = launch_simt_bwd_dq(*p, q, k, v, bs, lse, dsum, dout, dq, ws, tiles,
                         tile_capacity(*p, L.bm), st);
  if (e != cudaSuccess) return cuda_status(e);
  e = launch_simt_bwd_dkdv(*p, q, offsets, k, v, bs, lse, dsum, dout, dk, dv, ws, st);
  return cuda_status(e);
}

gdpa_status_t gdpa_bwd(const gdpa_problem_t* p, const void* q, const int32_t* offsets,
                       const void* k, const void* v, const void* o, const float* lse,
                       const void* dout, void* dq, void* dk, void* dv, void* workspace,
                       size_t workspace_bytes, void* stream) {
  return gdpa_bwd_bias(p, q, offsets, k, v, nullptr, nullptr, o, lse, dout, dq, dk, dv, nullptr,
                       nullptr, workspace, workspace_bytes, stream);
}

namespace {
// B <= 4096 (the pooling scheduler sorts the samples in one CTA's shared memory)
gdpa_status_t check_pool(int32_t B, int32_t h, int32_t dh, int32_t S, int64_t T, int32_t max_n,
                         float scale) {
  if (B < 1 || h < 1 || S < 1 || max_n < 0 || T < 0 || T >= (int64_t)1 << 31 ||
      (int64_t)max_n * B < T || !(scale == scale))
    return GDPA_ERR_INVALID_ARG;
  if ((dh != 32 && dh != 64) || S > 128 || B > 4096 || (int64_t)B * h >= (int64_t)1 << 24)
    return GDPA_ERR_UNSUPPORTED;
  return GDPA_OK;
}
size_t pool_ws_bytes(int32_t B, int32_t h) {
  return align_up(sizeof(WsHeader) + sizeof(Tile) * (size_t)B * ((h + 1) / 2), 256);
}
}  // namespace

gdpa_status_t gdpa_pool_workspace_size(int32_t B, int32_t h, int32_t dh, int32_t S,
                                       size_t* bytes) {
  const gdpa_status_t s = check_pool(B, h, dh, S, 0, 0, 1.f);
  if (s != GDPA_OK) return s;
  if (!bytes) return GDPA_ERR_INVALID_ARG;
  *bytes = pool_ws_bytes(B, h);
  return GDPA_OK;
}

gdpa_status_t gdpa_pool_fwd(int32_t B, int32_t h, int32_t dh, int32_t S, int64_t total_tokens,
                            int32_t max_n, float scale, const void* seeds,
                            const int32_t* offsets, const void* k, const void* v, void* o,
                            float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  g_launches = 0;
  gdpa_status_t s = check_pool(B, h, dh, S, total_tokens, max_n, scale);
  if (s != GDPA_OK) return s;
  const bool empty = total_tokens == 0;
  if (!offsets || !seeds || !o || (!empty && (!k || !v))) return GDPA_ERR_INVALID_ARG;
  if (!aligned16(seeds) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      ((uintptr_t)offsets & 3u) || ((uintptr_t)lse & 3u))
    return GDPA_ERR_INVALID_ARG;
  s = check_ws(workspace, workspace_bytes, pool_ws_bytes(B, h));
  if (s != GDPA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* ws = (WsHeader*)workspace;
  Tile* tiles = (Tile*)((char*)workspace + sizeof(WsHeader));
  cudaError_t e = launch_schedule_pool(offsets, B, h, total_tokens, max_n, ws, tiles, st);
  if (e == cudaSuccess) e = launch_pool_empty(offsets, B, h, S, dh, o, lse, ws, st);
  if (e == cudaSuccess)
    e = launch_sm100_pool(B, h, dh, S, total_tokens, scale, seeds, k, v, o, lse, ws, tiles, st);
  return cuda_status(e);
}

namespace {
gdpa_status_t check_window(int32_t B, int32_t h, int32_t dh, int64_t T, int32_t max_n,
                           int32_t window, float scale) {
  if (B < 1 || h < 1 || window < 1 || max_n < 0 || T < 0 || T >= (int64_t)1 << 31 ||
      (int64_t)max_n * B < T || !(scale == scale))
    return GDPA_ERR_INVALID_ARG;
  if ((dh != 32 && dh != 64) || (int64_t)B * h >= (int64_t)1 << 24) return GDPA_ERR_UNSUPPORTED;
  return GDPA_OK;
}
// the query-tile list of (h + 1) / 2 head pairs
gdpa_problem_t window_list_problem(int32_t B, int32_t h, int64_t T, int32_t max_n) {
  gdpa_problem_t p = {};
  p.B = B;
  p.h = (h + 1) / 2;
  p.dh = 64;
  p.m = 1;
  p.max_n = max_n;
  p.dtype = GDPA_DTYPE_BF16;
  p.total_tokens = T;
  p.phi = GDPA_PHI_SOFTMAX;
  p.scale = 1.f;
  return p;
}
}  // namespace

gdpa_status_t gdpa_window_workspace_size(int32_t B, int32_t h, int32_t dh, int64_t total_tokens,
                                         size_t* bytes) {
  const int32_t max_n = total_tokens >= 0 && total_tokens < 0x7fffffff ? (int32_t)total_tokens : 0;
  const gdpa_status_t s = check_window(B, h, dh, total_tokens, max_n, 1, 1.f);
  if (s != GDPA_OK) return s;
  if (!bytes) return GDPA_ERR_INVALID_ARG;
  const gdpa_problem_t lp = window_list_problem(B, h, total_tokens, 0);
  *bytes = align_up(sizeof(WsHeader) + sizeof(Tile) * (size_t)tile_capacity(lp, kMmaBM), 256);
  return GDPA_OK;
}

gdpa_status_t gdpa_window_fwd(int32_t B, int32_t h, int32_t dh, int64_t total_tokens,
                              int32_t max_n, int32_t window, float scale, const void* q,
                              const int32_t* offsets, const void* k, const void* v, void* o,
                              float* lse, void* workspace, size_t workspace_bytes, void* stream) {
  g_launches = 0;
  gdpa_status_t s = check_window(B, h, dh, total_tokens, max_n, window, scale);
  if (s != GDPA_OK) return s;
  const bool empty = total_tokens == 0;
  if (!offsets || (!empty && (!q || !k || !v || !o))) return GDPA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      ((uintptr_t)offsets & 3u) || ((uintptr_t)lse & 3u))
    return GDPA_ERR_INVALID_ARG;
  const gdpa_problem_t lp = window_list_problem(B, h, total_tokens, max_n);
  const size_t need =
      align_up(sizeof(WsHeader) + sizeof(Tile) * (size_t)tile_capacity(lp, kMmaBM), 256);
  s = check_ws(workspace, workspace_bytes, need);
  if (s != GDPA_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  WsHeader* ws = (WsHeader*)workspace;
  Tile* tiles = (Tile*)((char*)workspace + sizeof(WsHeader));
  cudaError_t e = launch_schedule(lp, offsets, kMmaBM, ws, tiles, st);
  if (e == cudaSuccess)
    e = launch_sm100_window(h, dh, total_tokens, window, scale, offsets, q, k, v, o, lse, ws,
                            tiles, st);
  return cuda_status(e);
}

namespace {
// backward work list of the jagged-key variants: h x (T / 128 + B) items at most
int64_t jkv_capacity(int32_t B, int32_t h, int64_t T) { return (int64_t)h * (T / 128 + B); }
size_t jkv_list_bytes(int32_t B, int32_t h, int64_t T) {
  return align_up(sizeof(WsHeader) + sizeof(Tile) * (size_t)jkv_capacity(B, h, T), 256);
}
// [list][dQ accumulator T x h x dh fp32][D h x T fp32]
size_t window_bwd_ws_bytes(int32_t B, int32_t h, int32_t dh, int64_t T) {
  return jkv_list_bytes(B, h, T) + align_up((size_t)T * h * dh * 4, 256) +
         align_up((size_t)T * h * 4, 256);
}
// [list][D B x h x S fp32]
size_t pool_bwd_ws_bytes(int32_t B, int32_t h, int32_t S, int64_t T) {
  return jkv_list_bytes(B, h, T) + align_up((size_t)B * h * S * 4, 256);
}
}  // namespace

gdpa_status_t gdpa_window_bwd_workspace_size(int32_t B, int32_t h, int32_t dh,
                                             int64_t total_tokens, size_t* bytes) {
  const int32_t max_n = total_tokens >= 0 && total_tokens < 0x7fffffff ? (int32_t)total_tokens : 0;
  gdpa_status_t s = check_window(B, h, dh, total_tokens, max_n, 1, 1.f);
  if (s != GDPA_OK) return s;
  if (B > 4096) return GDPA_ERR_UNSUPPORTED;
  if (!bytes) return GDPA_ERR_INVALID_ARG;
  *bytes = window_bwd_ws_bytes(B, h, dh, total_tokens);
  return GDPA_OK;
}

gdpa_status_t gdpa_window_bwd(int32_t B, int32_t h, int32_t dh, int64_t total_tokens,
                              int32_t max_n, int32_t window, float scale, const void* q,
                              const int32_t* offsets, const void* k, const void* v,
                              const void* o, const float* lse, const void* dout, void* dq,
                              void* dk, void* dv, void* workspace, size_t workspace_bytes,
                              void* stream) {
  g_launches = 0;
  gdpa_status_t s = check_window(B, h, dh, total_tokens, max_n, window, scale);
  if (s != GDPA_OK) return s;
  if (B > 4096) return GDPA_ERR_UNSUPPORTED;
  const bool empty = total_tokens == 0;
  if (!offsets || (!empty && (!q || !k || !v || !o || !lse || !dout || !dq || !dk || !dv)))
    return GDPA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || ((uintptr_t)offsets & 3u) ||
      ((uintptr_t)lse & 3u))
    return GDPA_ERR_INVALID_ARG;
  s = check_ws(workspace, workspace_bytes, window_bwd_ws_bytes(B, h, dh, total_tokens));
  if (s != GDPA_OK) return s;
  char* base = (char*)workspace;
  WsHeader* ws = (WsHeader*)base;
  Tile* tiles = (Tile*)(base + sizeof(WsHeader));
  float* dq_acc = (float*)(base + jkv_list_bytes(B, h, total_tokens));
  float* dsum = (float*)((char*)dq_acc + align_up((size_t)total_tokens * h * dh * 4, 256));
  return cuda_status(launch_sm100_window_bwd(
      B, h, dh, total_tokens, max_n, window, scale, offsets, q, k, v, o, lse, dout, dq, dk, dv,
      dq_acc, dsum, ws, tiles, jkv_capacity(B, h, total_tokens), (cudaStream_t)stream));
}

gdpa_status_t gdpa_pool_bwd_workspace_size(int32_t B, int32_t h, int32_t dh, int32_t S,
                                           int64_t total_tokens, size_t* bytes) {
  const gdpa_status_t s = check_pool(B, h, dh, S, 0, 0, 1.f);
  if (s != GDPA_OK) return s;
  if (!bytes || total_tokens < 0) return GDPA_ERR_INVALID_ARG;
  *bytes = pool_bwd_ws_bytes(B, h, S, total_tokens);
  return GDPA_OK;
}

gdpa_status_t gdpa_pool_bwd(int32_t B, int32_t h, int32_t dh, int32_t S, int64_t total_tokens,
                            int32_t max_n, float scale, const void* seeds,
                            const int32_t* offsets, const void* k, const void* v, const void* o,
                            const float* lse, const void* dout, float* dseeds, void* dk,
                            void* dv, void* workspace, size_t workspace_bytes, void* stream) {
  g_launches = 0;
  gdpa_status_t s = check_pool(B, h, dh, S, total_tokens, max_n, scale);
  if (s != GDPA_OK) return s;
  const bool empty = total_tokens == 0;
  if (!offsets || !seeds || !o || !lse || !dout || !dseeds || (!empty && (!k || !v || !dk || !dv)))
    return GDPA_ERR_INVALID_ARG;
  if (!aligned16(seeds) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dseeds) || !aligned16(dk) || !aligned16(dv) || ((uintptr_t)offsets & 3u) ||
      ((uintptr_t)lse & 3u))
    return GDPA_ERR_INVALID_ARG;
  s = check_ws(workspace, workspace_bytes, pool_bwd_ws_bytes(B, h, S, total_tokens));
  if (s != GDPA_OK) return s;
  char* base = (char*)workspace;
  WsHeader* ws = (WsHeader*)base;
  Tile* tiles = (Tile*)(base + sizeof(WsHeader));
  float* dsum = (float*)(base + jkv_list_bytes(B, h, total_tokens));
  return cuda_status(launch_sm100_pool_bwd(B, h, dh, S, total_tokens, max_n, scale, offsets,
                                           seeds, k, v, o, lse, dout, dseeds, dk, dv, dsum, ws,
                                           tiles, jkv_capacity(B, h, total_tokens),
                                           (cudaStream_t)stream));
}

gdpa_status_t gdpa_workspace_status(const void* workspace, void* stream, int32_t* status) {
  if (!workspace || !status) return GDPA_ERR_INVALID_ARG;
  int32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost,
                                  (cudaStream_t)stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_status(e);
  *status = v;
  return GDPA_OK;
}

const char* gdpa_status_string(gdpa_status_t s) {
  switch (s) {
    case GDPA_OK: return "GDPA_OK";
    case GDPA_ERR_INVALID_ARG: return "GDPA_ERR_INVALID_ARG: invalid argument or offsets";
    case GDPA_ERR_UNSUPPORTED: return "GDPA_ERR_UNSUPPORTED: unsupported problem shape";
    case GDPA_ERR_CUDA: return "GDPA_ERR_CUDA: CUDA call or kernel launch failed";
    case GDPA_ERR_TIMEOUT: return "GDPA_ERR_TIMEOUT: a bounded wait inside a kernel expired";
    case GDPA_ERR_WORKSPACE: return "GDPA_ERR_WORKSPACE: workspace null, misaligned or too small";
  }
  return "GDPA: unknown status";
}

int32_t gdpa_last_launch_count(void) { return g_launches; }

gdpa_status_t gdpa_timing_enable(int32_t enable) {
  clear_records();
  g_timing = enable != 0;
  return GDPA_OK;
}

int32_t gdpa_timing_read(gdpa_kernel_time_t* out, int32_t cap) {
  std::vector<std::string> names;
  std::vector<int> counts;
  std::vector<float> totals;
  for (auto& r : g_recs) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) {
      clear_records();
      return -1;
    }
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
      clear_records();
      return -1;
    }
    size_t i = 0;
    while (i < names.size() && names[i] != r.name) ++i;
    if (i == names.size()) {
      names.push_back(r.name);
      counts.push_back(0);
      totals.push_back(0.f);
    }
    counts[i] += 1;
    totals[i] += ms;
  }
  clear_records();
  for (size_t i = 0; i < names.size() && (int32_t)i < cap && out; ++i) {
    memset(out[i].name, 0, sizeof(out[i].name));
    strncpy(out[i].name, names[i].c_str(), sizeof(out[i].name) - 1);
    out[i].launches = counts[i];
    out[i].total_ms = totals[i];
  }
  return (int32_t)names.size();
}

}  // extern "C"
