// Self-test of the device-side failure path shared by the GDPA kernels: a
// bounded mbarrier wait that gives up, records GDPA_ERR_TIMEOUT in the
// workspace status word and returns, leaving the CUDA context usable.
#include "gdpa_internal.cuh"
#include "sm100.cuh"

namespace gdpa {
namespace {

__global__ void wait_timeout_kernel(WsHeader* ws, uint64_t timeout_ns) {
  __shared__ uint64_t never_completed;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ws->status = GDPA_OK;
    sm100::mbar_init(sm100::smem_u32(&never_completed), 1);   // nothing ever arrives
    sm100::fence_mbar_init();
    abort_flag = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool done = sm100::mbar_wait(sm100::smem_u32(&never_completed), 0,
                                       reinterpret_cast<volatile int*>(&abort_flag), timeout_ns);
    if (!done) report(ws, GDPA_ERR_TIMEOUT);
  }
}

}  // namespace
}  // namespace gdpa

extern "C" gdpa_status_t gdpa_selftest_wait_timeout(void* workspace, size_t workspace_bytes,
                                                    uint32_t timeout_us, void* stream) {
  if (!workspace || ((uintptr_t)workspace & 255u) || workspace_bytes < sizeof(gdpa::WsHeader) ||
      timeout_us == 0 || timeout_us > 5000000u)
    return GDPA_ERR_INVALID_ARG;
  {
    gdpa::KernelScope ks_("gdpa_selftest_wait_timeout", (cudaStream_t)stream);
    gdpa::wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(
        reinterpret_cast<gdpa::WsHeader*>(workspace), 1000ull * timeout_us);
  }
  return cudaGetLastError() == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}
