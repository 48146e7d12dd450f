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

namespace gdpa {
namespace {

// y_fma[i] = exp2_fma2(x[i]) (the FMA-pipe exp2 of the softmax kernels) and
// y_mufu[i] = ex2.approx.ftz (the MUFU unit), for checking the former against
// a reference exp2 and against the latter.
__global__ void exp2_selftest_kernel(const float* __restrict__ x, float* __restrict__ y_fma,
                                     float* __restrict__ y_mufu, int64_t n) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const float v = x[i];
    y_fma[i] = exp2_fma2(make_float2(v, v)).x;
    y_mufu[i] = sm100::ex2_approx(v);
  }
}

}  // namespace
}  // namespace gdpa

extern "C" gdpa_status_t gdpa_selftest_exp2(const float* x, float* y_fma, float* y_mufu,
                                            int64_t n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y_fma || !y_mufu))) return GDPA_ERR_INVALID_ARG;
  if (n == 0) return GDPA_OK;
  const int64_t blocks = (n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184;
  {
    gdpa::KernelScope ks_("gdpa_selftest_exp2", (cudaStream_t)stream);
    gdpa::exp2_selftest_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(x, y_fma,
                                                                                   y_mufu, n);
  }
  return cudaGetLastError() == cudaSuccess ? GDPA_OK : GDPA_ERR_CUDA;
}
