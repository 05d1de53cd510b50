// gemm_tc.cu -- tensor-core prefill GEMM (placeholder until the tcgen05 kernel lands).
#include "tq_internal.cuh"

namespace tq {
cudaError_t launch_gemm_tc(const uint16_t*, int64_t, const uint8_t*, const uint16_t*, int64_t,
                           int64_t, int, void*, int, uint32_t*, cudaStream_t, int, bool* handled) {
    *handled = false;
    return cudaSuccess;
}
}  // namespace tq
