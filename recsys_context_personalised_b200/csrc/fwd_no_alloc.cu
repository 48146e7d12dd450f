// gdpa_fwd_no_alloc: the GDPA forward with its scratch memory in a static
// device array, for callers that cannot allocate device memory when they call
// the operator.  Examples: a host framework that reserves all device memory
// for its own pool at start-up and gives plug-in operators no allocator, or a
// latency-bound serving loop in which cudaMalloc's implicit synchronisation is
// not acceptable.  Such a caller passes only inputs and outputs.
//
// The scratch is what gdpa_fwd keeps in its workspace: a 256-byte header
// (device status word, tile count) and the jagged tile list.  It lives in
// `g_fwd_scratch` below, kFwdScratchBytes (2 MiB) per device that loads the
// library, held until the process exits.
#include <mutex>

#include "gdpa_internal.cuh"

namespace gdpa {
namespace {

constexpr size_t kFwdScratchBytes = 2u << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_fwd_scratch[kFwdScratchBytes];

// Device addresses of g_fwd_scratch, one per device, filled on first use.
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

// Set-up, once per device and with that device current: in host code the
// array's name is only a host-side stand-in, so its device address has to be
// queried.  Returns nullptr on failure.
void* scratch_address(int dev) {
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (!g_scratch_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_fwd_scratch) != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
  }
  return g_scratch_addr[dev];
}

}  // namespace
}  // namespace gdpa

extern "C" gdpa_status_t gdpa_fwd_no_alloc(const gdpa_problem_t* p, const void* q,
                                           const int32_t* offsets, const void* k, const void* v,
                                           void* o, float* lse, void* stream) {
  size_t need = 0;
  gdpa_status_t s = gdpa_fwd_workspace_size(p, &need);
  if (s != GDPA_OK) return s;
  if (need > gdpa::kFwdScratchBytes) return GDPA_ERR_WORKSPACE;   // beyond the static maximum
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= gdpa::kMaxDevices)
    return GDPA_ERR_CUDA;
  void* scratch = gdpa::scratch_address(dev);
  if (!scratch) return GDPA_ERR_CUDA;
  // Nothing in the scratch has to start at zero: the scheduling kernel
  // rewrites the header and the tile list at the start of every call.
  return gdpa_fwd(p, q, offsets, k, v, o, lse, scratch, gdpa::kFwdScratchBytes, stream);
}

// Device-detected status of the last gdpa_fwd_no_alloc call on the current
// device (the header's status word in the static scratch): GDPA_OK, or
// GDPA_ERR_INVALID_ARG for inconsistent device offsets, or GDPA_ERR_TIMEOUT.
// Copies four bytes on `stream` and synchronises it; allocates nothing.
extern "C" gdpa_status_t gdpa_fwd_no_alloc_status(void* stream, int32_t* status) {
  if (!status) return GDPA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= gdpa::kMaxDevices)
    return GDPA_ERR_CUDA;
  void* scratch = gdpa::scratch_address(dev);
  if (!scratch) return GDPA_ERR_CUDA;
  return gdpa_workspace_status(scratch, stream, status);
}
