// noalloc.cu -- nf4_lora_linear_fwd_noalloc: the fused LoRA linear for
// callers that cannot allocate device memory.
//
// nf4_lora_linear_fwd needs a caller-provided workspace for the low-rank
// intermediate t.  Some callers have no way to provide one: a plugin that is
// handed only its input and output buffers and holds no allocator, a serving
// loop that must not call cudaMalloc (which may synchronize the whole device)
// in the middle of a latency-critical step, or a framework whose memory is
// fully reserved by its own pool.  This entry point takes the same inputs and
// outputs and keeps t in a fixed scratch array that lives in this file.
//
// The scratch is a file-scope __device__ array of NF4_NOALLOC_SCRATCH_BYTES
// (4 MiB); every GPU that loads the library holds it until the process exits.
// Its name is only a host-side handle in host code, so the device address is
// looked up with cudaGetSymbolAddress once per device, on that device's first
// call (with that device current) -- make that first call before any stream
// capture begins.  All calls on a device share the one array and it keeps the
// previous call's contents; the down-projection kernel rewrites every byte the
// linear reads (including the zero padding columns) on each call, so nothing
// has to be cleared in advance.  Two calls whose kernels overlap on the GPU
// (different streams without ordering) race on the array and give undefined
// results.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "../../include/nf4.h"
#include "nf4_device.cuh"

namespace nf4 {
cudaError_t launch_lora_linear(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed,
                               const uint8_t *q8, const float *scales, const float *offset, const void *A,
                               const void *B, int r, float scaling, void *y, void *workspace,
                               int64_t workspace_bytes, cudaStream_t stream, int num_sms, unsigned *err_word);
int64_t lora_workspace_bytes(int64_t M, int r);
int64_t linear_workspace_bytes(int64_t M, int r);
unsigned *device_error_word(cudaError_t *status);
nf4_status status_of(cudaError_t e);
}  // namespace nf4

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[NF4_NOALLOC_SCRATCH_BYTES];

std::mutex g_setup_mutex;
void *g_scratch_ptr[64] = {nullptr};
int g_sm_count[64] = {0};

// Device address of the scratch array and the SM count of the current device,
// looked up on the first call per device.
cudaError_t scratch_for_current_device(void **ptr, int *sms) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        int v = 0;
        e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        g_sm_count[dev] = v;
        g_scratch_ptr[dev] = p;
    }
    *ptr = g_scratch_ptr[dev];
    *sms = g_sm_count[dev];
    return cudaSuccess;
}

bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" NF4_API nf4_status nf4_lora_linear_fwd_noalloc(const void *x, int64_t M, int64_t K, int64_t N,
                                                           const uint8_t *packed, const uint8_t *absmax_q,
                                                           const float *absmax2, const float *offset,
                                                           const void *A, const void *B, int r, float scaling,
                                                           void *y, void *stream) {
    if (M < 1 || N < 1 || K < nf4::kBlock || (K % nf4::kBlock) != 0) return NF4_ERR_INVALID;
    if (r != 0 && r != 16 && r != 32 && r != 64) return NF4_ERR_UNSUPPORTED;
    if (!x || !packed || !absmax2 || !y) return NF4_ERR_INVALID;
    if (absmax_q == nullptr && offset != nullptr) return NF4_ERR_INVALID;
    const bool lora = (r > 0 && A != nullptr && B != nullptr);
    if (!aligned16(x) || !aligned16(packed) || !aligned16(absmax_q) || !aligned16(absmax2) || !aligned16(offset) ||
        !aligned16(y) || !aligned16(A) || !aligned16(B))
        return NF4_ERR_INVALID;
    if ((N % 8) != 0) return NF4_ERR_UNSUPPORTED;
    if (lora && nf4::lora_workspace_bytes(M, r) > (int64_t)NF4_NOALLOC_SCRATCH_BYTES)
        return NF4_ERR_UNSUPPORTED;  // the intermediate does not fit the fixed scratch
    void *scratch = nullptr;
    int sms = 0;
    cudaError_t e = scratch_for_current_device(&scratch, &sms);
    if (e == cudaSuccess) {
        unsigned *err = nf4::device_error_word(&e);
        if (e == cudaSuccess)
            e = nf4::launch_lora_linear(x, M, K, N, packed, absmax_q, absmax2, offset, lora ? A : nullptr,
                                        lora ? B : nullptr, lora ? r : 0, scaling, y, scratch,
                                        (int64_t)NF4_NOALLOC_SCRATCH_BYTES, (cudaStream_t)stream, sms, err);
    }
    return nf4::status_of(e);
}
