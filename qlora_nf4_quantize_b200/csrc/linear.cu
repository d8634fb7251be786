// linear.cu -- dispatch of the fused frozen-base LoRA linear, its workspace
// layout, and the device error word written by kernels whose bounded waits
// expire.
#include <mutex>

#include "nf4_device.cuh"

namespace nf4 {

int lora_rp(int r);
cudaError_t launch_lora_down(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2,
                             unsigned *counts, int ncounts, cudaStream_t stream);
cudaError_t launch_decode(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                          const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                          void *y, unsigned *err, cudaStream_t stream, int num_sms);
cudaError_t launch_lora_down_tc(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2, int rp,
                                unsigned *err, cudaStream_t stream, int split, int max_ctas);
cudaError_t launch_gemm_tc(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                           const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                           void *y, float *partials, unsigned *counts, int ctas, cudaStream_t stream,
                           unsigned *err_word);
int64_t streamk_partials_bytes();
int64_t streamk_counts_bytes();
int streamk_ctas(int64_t M, int64_t K, int64_t N, int rp, int sms);

constexpr int kGemvMaxTokens = 16;
// Token counts from which decode-size calls take the tcgen05 pipeline with a
// 16-token tile, split over the SMs, instead of the warp-MMA decode kernel
// (decode.cu: up to 16 tokens).  The default (17) sends every decode-size
// call to the decode kernel, which is faster at every count (at 16 tokens,
// W 11008 x 4096, r = 16: 22.6 against 26.0 us); a build with 9 keeps the
// split pipeline for 9..16 tokens.
#ifndef NF4_SMALL_M_TC_FROM
#define NF4_SMALL_M_TC_FROM 17
#endif
static_assert(NF4_SMALL_M_TC_FROM >= 9 && NF4_SMALL_M_TC_FROM <= 17, "the decode kernel serves 1..8 tokens at least, 16 at most");

// Device error word: one per device, cleared by nf4_device_status().  Its
// device address is looked up once per device (with that device current)
// and cached for the life of the process's context on that device; the
// cache is guarded so that host threads making their first calls at the
// same time do not race on it.
static __device__ unsigned g_error_word;

unsigned *device_error_word(cudaError_t *status) {
    static std::mutex mutex;
    static unsigned *cached[64] = {nullptr};
    int dev = 0;
    *status = cudaGetDevice(&dev);
    if (*status != cudaSuccess) return nullptr;
    if (dev < 0 || dev >= 64) {
        *status = cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mutex);
    if (cached[dev] == nullptr) {
        void *p = nullptr;
        *status = cudaGetSymbolAddress(&p, g_error_word);
        if (*status != cudaSuccess) return nullptr;
        cached[dev] = static_cast<unsigned *>(p);
    }
    return cached[dev];
}

// t2 = [t_hi | t_lo | 0 pad] bf16 [M, round_up(2r, 64)], 16-byte aligned rows.
int64_t lora_workspace_bytes(int64_t M, int r) { return M * (int64_t)lora_rp(r) * 2; }

// Token counts served by the split 16-token pipeline (none in the default
// build): for them the workspace continues (256-byte aligned) with its
// scratch, partial tiles then arrival counts.  A workspace holding only t (or
// none, r = 0) runs it unsplit.
static bool split_tokens(int64_t M) { return M >= NF4_SMALL_M_TC_FROM && M <= kGemvMaxTokens; }
static int64_t partials_offset(int64_t M, int r) {
    return (lora_workspace_bytes(M, r > 0 ? r : 0) + 255) & ~(int64_t)255;
}
int64_t linear_workspace_bytes(int64_t M, int r) {
    if (split_tokens(M)) return partials_offset(M, r) + streamk_partials_bytes() + streamk_counts_bytes();
    return r > 0 ? lora_workspace_bytes(M, r) : 0;
}

// The arrival counts of a split launch without an adapter are zeroed by
// this one-CTA kernel, which keeps the chain of programmatic dependent
// launches: it waits for the grid before it (the previous call, which may
// still use the counts), zeroes them and releases the linear.
__global__ void k_zero_counts(unsigned *counts, int n) {
    pdl_wait_then_release();
    for (int i = threadIdx.x; i < n; i += blockDim.x) counts[i] = 0u;
}

cudaError_t launch_lora_linear(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed,
                               const uint8_t *q8, const float *scales, const float *offset, const void *A,
                               const void *B, int r, float scaling, void *y, void *workspace,
                               int64_t workspace_bytes, cudaStream_t stream, int num_sms, unsigned *err_word) {
    const int rp = r > 0 ? lora_rp(r) : 0;
    // decode-size M: the warp-MMA decode kernel up to NF4_SMALL_M_TC_FROM - 1
    // tokens, then the tcgen05 pipeline with a 16-token tile, split over the
    // SMs when the workspace holds its scratch (with an adapter, 8 SMs are
    // left to the down-projection's cluster, which runs first)
    const bool gemv = M < NF4_SMALL_M_TC_FROM;
    float *partials = nullptr;
    unsigned *counts = nullptr;
    int ctas = 0;
    if (split_tokens(M) && workspace != nullptr && workspace_bytes >= linear_workspace_bytes(M, r)) {
        ctas = streamk_ctas(M, K, N, rp, r > 0 && num_sms > 16 ? num_sms - 8 : num_sms);
        if (ctas > 0) {
            partials = reinterpret_cast<float *>(static_cast<char *>(workspace) + partials_offset(M, r));
            counts = reinterpret_cast<unsigned *>(reinterpret_cast<char *>(partials) + streamk_partials_bytes());
        }
    }
    const int ncounts = ctas > 0 ? (int)((N + 127) / 128) : 0;
    cudaError_t e = cudaSuccess;
    if (r > 0) {
        // decode-size M: warp-MMA kernel; larger M: tensor-core kernel
        // with fewer GEMM tiles than SMs (a small N), the down-projection is
        // held to the SMs the GEMM leaves idle, so that no GEMM tile waits
        // for an SM it holds (one CTA per 128-row tile otherwise)
        const int64_t gemm_ctas = ((N + 127) / 128) * ((M + 255) / 256);
        const int idle = gemm_ctas < num_sms ? num_sms - (int)gemm_ctas : 0;
        e = M <= kGemvMaxTokens
                ? launch_lora_down(x, A, M, K, r, scaling, workspace, counts, ncounts, stream)
                : launch_lora_down_tc(x, A, M, K, r, scaling, workspace, rp, err_word, stream, 0, idle >= 8 ? idle : 0);
    } else if (ctas > 0) {
        e = launch_pdl(k_zero_counts, dim3(1), dim3(256), 0, stream, 1, counts, ncounts);
    }
    if (e != cudaSuccess) return e;
    // with an adapter, the 8 SMs of the down-projection's cluster (launched
    // just before) are left to it
    if (gemv)
        return launch_decode(x, (int)M, K, N, packed, q8, scales, offset, B, r, workspace, rp, y, err_word, stream,
                             r > 0 && num_sms > 16 ? num_sms - 8 : num_sms);
    return launch_gemm_tc(x, M, K, N, packed, q8, scales, offset, B, r, workspace, rp, y, partials, counts, ctas, stream,
                          err_word);
}

}  // namespace nf4
