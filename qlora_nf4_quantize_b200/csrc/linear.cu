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
// Token counts from which decode-size calls take the tcgen05 pipeline with a
// 16-token tile instead of the warp-MMA GEMV kernels: that pipeline takes
// the same time for any count up to 16 (25.7 us without LoRA on an 11008 x
// 4096 weight), the warp-MMA kernels grow with it (17.0 us at 1 token, 21.8
// at 8, 27.5 at 12, 30.3 at 16: above 8 tokens they need two token tiles).
#ifndef NF4_SMALL_M_TC_FROM
#define NF4_SMALL_M_TC_FROM 9
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
    // decode-size M: the warp-MMA GEMV kernels up to NF4_SMALL_M_TC_FROM - 1
    // tokens, then the tcgen05 pipeline with a 16-token tile
    if (M < NF4_SMALL_M_TC_FROM && M <= kGemvMaxTokens)
        return launch_gemv(x, (int)M, K, N, packed, q8, scales, offset, B, r, workspace, rp, y, stream, num_sms);
    return launch_gemm_tc(x, M, K, N, packed, q8, scales, offset, B, r, workspace, rp, y, stream, num_sms,
                          err_word);
}

}  // namespace nf4
