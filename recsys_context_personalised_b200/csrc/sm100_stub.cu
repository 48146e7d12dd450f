// Placeholder for the tcgen05 backward until it is compiled in.
#include "gdpa_internal.cuh"

namespace gdpa {
bool sm100_bwd_available() { return false; }
cudaError_t launch_sm100_bwd(const gdpa_problem_t&, const void*, const int32_t*, const void*,
                             const void*, const float*, const float*, const void*, void*, void*,
                             void*, float*, WsHeader*, const Tile*, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace gdpa
