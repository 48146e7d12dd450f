// Placeholder for the tcgen05 kernels until they are compiled in.
#include "gdpa_internal.cuh"

namespace gdpa {
bool sm100_fwd_available() { return false; }
bool sm100_bwd_available() { return false; }
cudaError_t launch_sm100_fwd(const gdpa_problem_t&, const void*, const void*, const void*, void*,
                             float*, WsHeader*, const Tile*, cudaStream_t) {
  return cudaErrorNotSupported;
}
cudaError_t launch_sm100_bwd(const gdpa_problem_t&, const void*, const int32_t*, const void*,
                             const void*, const float*, const float*, const void*, void*, void*,
                             void*, float*, WsHeader*, const Tile*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace gdpa
