// gemm_w4a8.cu -- W4A8 tensor-core GEMM (placeholder until the kernel lands).
#include "qk_internal.h"

namespace qk {
cudaError_t launch_w4a8_gemm(const int8_t*, const float*, const int32_t*, int64_t, int64_t,
                             const uint8_t*, const uint16_t*, const uint16_t*, const float*,
                             int64_t, uint16_t*, int32_t*, int64_t, int64_t, bool, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace qk
