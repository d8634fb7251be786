// linear.cu -- dispatch of the fused frozen-base LoRA linear, its workspace
// layout, and the device error word written by kernels whose bounded waits
// expire.
#include "nf4_device.cuh"

namespace nf4 {

int lora_rp(int r);
cudaError_t launch_lora_down(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2,
                             cudaStream_t stream);
cudaError_t launch_gemv(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                        const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                        void *y, cudaStream_t stream, int num_sms);
cudaError_t launch_lora_down_tc(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2, int rp,
                                unsigned *err, cudaStream_t stream, int split);
cudaError_t launch_gemm_tc(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                           const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                           void *y, cudaStream_t stream, int num_sms, unsigned *err_word);

constexpr int kGemvMaxTokens = 16;
#ifndef NF4_SMALL_M_TC
#define NF4_SMALL_M_TC 0
#endif

// Device error word: one per device, cleared by nf4_device_status().
static __device__ unsigned g_error_word;

unsigned *device_error_word(cudaError_t *status) {
    static unsigned *cached[64] = {nullptr};
    int dev = 0;
    *status = cudaGetDevice(&dev);
    if (*status != cudaSuccess) return nullptr;
    if (dev >= 0 && dev < 64 && cached[dev] != nullptr) return cached[dev];
    void *p = nullptr;
    *status = cudaGetSymbolAddress(&p, g_error_word);
    if (*status != cudaSuccess) return nullptr;
    if (dev >= 0 && dev < 64) cached[dev] = static_cast<unsigned *>(p);
    return static_cast<unsigned *>(p);
}

// t2 = [t_hi | t_lo | 0 pad] bf16 [M, round_up(2r, 64)], 16-byte aligned rows.
int64_t lora_workspace_bytes(int64_t M, int r) { return M * (int64_t)lora_rp(r) * 2; }

cudaError_t launch_lora_linear(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed,
                               const uint8_t *q8, const float *scales, const float *offset, const void *A,
                               const void *B, int r, float scaling, void *y, void *workspace,
                               cudaStream_t stream, int num_sms, unsigned *err_word) {
    const int rp = r > 0 ? lora_rp(r) : 0;
    if (r > 0) {
        // decode-size M: warp-MMA kernel; larger M: tensor-core kernel
        cudaError_t e = M <= kGemvMaxTokens ? launch_lora_down(x, A, M, K, r, scaling, workspace, stream)
                                            : launch_lora_down_tc(x, A, M, K, r, scaling, workspace, rp, err_word, stream, 0);
        if (e != cudaSuccess) return e;
    }
    // decode-size M: the warp-MMA GEMV kernels, or (built with
    // NF4_SMALL_M_TC=1) the tcgen05 pipeline with a 16-token tile
    if (M <= kGemvMaxTokens && !NF4_SMALL_M_TC)
        return launch_gemv(x, (int)M, K, N, packed, q8, scales, offset, B, r, workspace, rp, y, stream, num_sms);
    return launch_gemm_tc(x, M, K, N, packed, q8, scales, offset, B, r, workspace, rp, y, stream, num_sms,
                          err_word);
}

}  // namespace nf4
