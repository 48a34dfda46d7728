// KDA chunked prefill on the tcgen05 tensor cores (placeholder until the kernel lands).
#include "kda_common.cuh"

namespace kda {
bool prefill_tc_supported(int, int, int, int) { return false; }
cudaError_t launch_prefill_tc(const void *, const void *, const void *, const float *,
                              const float *, const float *, const int32_t *, void *, float *,
                              int64_t, float *, int, int, int64_t, int32_t *, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace kda
