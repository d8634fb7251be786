// gemm_tc.cu -- K5: fused NF4-dequantizing tensor-core GEMM (tcgen05) for
// large token counts.  (Implementation in progress.)
#include "nf4_device.cuh"

namespace nf4 {

cudaError_t launch_gemm_tc(const void *, int64_t, int64_t, int64_t, const uint8_t *, const uint8_t *,
                           const float *, const float *, const void *, int, const void *, int, void *,
                           cudaStream_t, int, unsigned *) {
    return cudaErrorNotSupported;
}

}  // namespace nf4
