// capi.cu -- the extern "C" entry points of libnf4.so (declared and
// documented in include/nf4.h): argument validation, launch configuration and
// CUDA error mapping.  All arithmetic is in the kernels.
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include <atomic>

#include "../../include/nf4.h"
#include "nf4_device.cuh"

namespace nf4 {
cudaError_t launch_quantize(const void *w, bool bf16, int64_t n, uint8_t *packed, float *absmax,
                            cudaStream_t stream, int num_sms);
int64_t dq_run_count(int64_t nblocks);
int64_t dq_chunk_count(int64_t nblocks);
int64_t dq_max_chunks();
int64_t dq_workspace_bytes(int64_t nblocks);
cudaError_t launch_double_quantize(const float *absmax, int64_t nb, uint8_t *codes, float *absmax2,
                                   float *offset, double *workspace, cudaStream_t stream, int num_sms);
cudaError_t launch_dq_run_sums(const float *absmax, int64_t nb, double *run_sums, cudaStream_t stream);
cudaError_t launch_dq_from_run_sums(const float *absmax, int64_t nb, const double *run_sums, int64_t nb_total,
                                    uint8_t *codes, float *absmax2, float *offset, double *chunk_sums,
                                    cudaStream_t stream, int num_sms);
cudaError_t launch_dequantize(const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                              int64_t n, void *out, bool bf16, cudaStream_t stream, int num_sms);
cudaError_t launch_lora_linear(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed,
                               const uint8_t *q8, const float *scales, const float *offset, const void *A,
                               const void *B, int r, float scaling, void *y, void *workspace,
                               int64_t workspace_bytes, cudaStream_t stream, int num_sms, unsigned *err_word);
int64_t lora_workspace_bytes(int64_t M, int r);
int64_t linear_workspace_bytes(int64_t M, int r);
unsigned *device_error_word(cudaError_t *status);
cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t stream);
cudaError_t launch_merge_requantize(const uint8_t *packed, const uint8_t *q8, const float *scales,
                                    const float *offset, int64_t N, int64_t K, const void *A, const void *B, int r,
                                    float s, uint8_t *packed_out, float *absmax_out, cudaStream_t stream);
int merge_max_rank();
int64_t lora_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int r);
cudaError_t launch_lora_linear_bwd(const void *g, const void *x, int64_t M, int64_t K, int64_t N,
                                   const uint8_t *packed, const uint8_t *q8, const float *scales,
                                   const float *offset, const void *A, const void *B, int r, float s, void *dx,
                                   float *dA, float *dB, void *workspace, unsigned *err, cudaStream_t stream,
                                   int num_sms);
}  // namespace nf4

namespace {

std::atomic<int> g_last_cuda_error{0};

nf4_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return NF4_OK;
    g_last_cuda_error.store((int)e);
    return NF4_ERR_CUDA;
}

bool aligned16(const void *p) { return p == nullptr || ((uintptr_t)p & 15u) == 0; }

// SM count of the current device, cached per device (atomic entries: host
// threads making their first calls at the same time write the same value).
int sm_count(cudaError_t *status) {
    static std::atomic<int> cached[64];
    int dev = 0;
    *status = cudaGetDevice(&dev);
    if (*status != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int v = 0;
    *status = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    if (*status != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) cached[dev].store(v, std::memory_order_relaxed);
    return v;
}

}  // namespace

namespace nf4 {
// Status mapping shared with entry points defined in other files.
nf4_status status_of(cudaError_t e) { return cuda_status(e); }
}  // namespace nf4

extern "C" {

const char *nf4_status_string(nf4_status s) {
    switch (s) {
        case NF4_OK: return "NF4_OK";
        case NF4_ERR_INVALID: return "NF4_ERR_INVALID";
        case NF4_ERR_UNSUPPORTED: return "NF4_ERR_UNSUPPORTED";
        case NF4_ERR_CUDA: return "NF4_ERR_CUDA";
        case NF4_ERR_TIMEOUT: return "NF4_ERR_TIMEOUT";
    }
    return "NF4_ERR_UNKNOWN";
}

int nf4_last_cuda_error(void) { return g_last_cuda_error.load(); }

nf4_status nf4_codebook(float *out_host) {
    if (out_host == nullptr) return NF4_ERR_INVALID;
    memcpy(out_host, nf4::kLevelsHost, sizeof nf4::kLevelsHost);
    return NF4_OK;
}

nf4_status nf4_quantize(const void *w, nf4_dtype w_dtype, int64_t n, int blocksize, uint8_t *packed,
                        float *absmax, void *stream) {
    if (blocksize != nf4::kBlock) return NF4_ERR_UNSUPPORTED;
    if (n < 0 || (n & 1) || (w_dtype != NF4_F32 && w_dtype != NF4_BF16)) return NF4_ERR_INVALID;
    if (n == 0) return NF4_OK;
    if (!w || !packed || !absmax || !aligned16(w) || !aligned16(packed) || !aligned16(absmax)) return NF4_ERR_INVALID;
    cudaError_t st;
    int sms = sm_count(&st);
    if (st != cudaSuccess) return cuda_status(st);
    return cuda_status(nf4::launch_quantize(w, w_dtype == NF4_BF16, n, packed, absmax, (cudaStream_t)stream, sms));
}

// Workspace of nf4_quantize_dq: the fp32 first-level constants (256-byte
// aligned), then the run sums and chunk sums of the centring mean.
static int64_t qdq_absmax_bytes(int64_t nb) { return (nb * 4 + 255) & ~(int64_t)255; }

int64_t nf4_quantize_dq_workspace_size(int64_t n, int blocksize, int dq_blocksize) {
    if (n <= 0 || blocksize != nf4::kBlock || dq_blocksize != nf4::kDqBlock) return 0;
    const int64_t nb = (n + nf4::kBlock - 1) / nf4::kBlock;
    return qdq_absmax_bytes(nb) + nf4::dq_workspace_bytes(nb);
}

nf4_status nf4_quantize_dq(const void *w, nf4_dtype w_dtype, int64_t n, int blocksize, int dq_blocksize,
                           uint8_t *packed, uint8_t *absmax_q, float *absmax2, float *offset, void *workspace,
                           int64_t workspace_bytes, void *stream) {
    if (blocksize != nf4::kBlock || dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
    if (n < 0 || (n & 1) || (w_dtype != NF4_F32 && w_dtype != NF4_BF16)) return NF4_ERR_INVALID;
    if (n == 0) return NF4_OK;
    if (!w || !packed || !absmax_q || !absmax2 || !workspace) return NF4_ERR_INVALID;
    if (!aligned16(w) || !aligned16(packed) || !aligned16(absmax_q) || !aligned16(absmax2) || !aligned16(offset) ||
        ((uintptr_t)workspace & 255u) != 0)
        return NF4_ERR_INVALID;
    if (workspace_bytes < nf4_quantize_dq_workspace_size(n, blocksize, dq_blocksize)) return NF4_ERR_INVALID;
    const int64_t nb = (n + nf4::kBlock - 1) / nf4::kBlock;
    if (offset != nullptr && nf4::dq_chunk_count(nb) > nf4::dq_max_chunks()) return NF4_ERR_UNSUPPORTED;
    cudaError_t st;
    int sms = sm_count(&st);
    if (st != cudaSuccess) return cuda_status(st);
    float *c1 = static_cast<float *>(workspace);
    double *sums = reinterpret_cast<double *>(static_cast<char *>(workspace) + qdq_absmax_bytes(nb));
    st = nf4::launch_quantize(w, w_dtype == NF4_BF16, n, packed, c1, (cudaStream_t)stream, sms);
    if (st != cudaSuccess) return cuda_status(st);
    return cuda_status(
        nf4::launch_double_quantize(c1, nb, absmax_q, absmax2, offset, sums, (cudaStream_t)stream, sms));
}

int64_t nf4_double_quantize_workspace_size(int64_t nblocks, int dq_blocksize) {
    if (nblocks <= 0 || dq_blocksize != nf4::kDqBlock) return 0;
    return nf4::dq_workspace_bytes(nblocks);
}

nf4_status nf4_double_quantize(const float *absmax, int64_t nblocks, int dq_blocksize, uint8_t *absmax_q,
                               float *absmax2, float *offset, void *workspace, int64_t workspace_bytes,
                               void *stream) {
    if (dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
    if (nblocks < 0) return NF4_ERR_INVALID;
    if (nblocks == 0) return NF4_OK;
    if (!absmax || !absmax_q || !absmax2) return NF4_ERR_INVALID;
    if (!aligned16(absmax) || !aligned16(absmax_q) || !aligned16(absmax2) || !aligned16(offset) ||
        !aligned16(workspace))
        return NF4_ERR_INVALID;
    if (offset != nullptr) {
        if (nf4::dq_chunk_count(nblocks) > nf4::dq_max_chunks()) return NF4_ERR_UNSUPPORTED;
        if (workspace == nullptr || workspace_bytes < nf4_double_quantize_workspace_size(nblocks, dq_blocksize))
            return NF4_ERR_INVALID;
    }
    cudaError_t st;
    int sms = sm_count(&st);
    if (st != cudaSuccess) return cuda_status(st);
    return cuda_status(nf4::launch_double_quantize(absmax, nblocks, absmax_q, absmax2, offset,
                                                   static_cast<double *>(workspace), (cudaStream_t)stream, sms));
}

nf4_status nf4_dq_run_sums(const float *absmax, int64_t nblocks, int dq_blocksize, double *run_sums,
                           void *stream) {
    if (dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
    if (nblocks < 0) return NF4_ERR_INVALID;
    if (nblocks == 0) return NF4_OK;
    if (!absmax || !run_sums || !aligned16(absmax) || !aligned16(run_sums)) return NF4_ERR_INVALID;
    return cuda_status(nf4::launch_dq_run_sums(absmax, nblocks, run_sums, (cudaStream_t)stream));
}

int64_t nf4_double_quantize_sharded_workspace_size(int64_t nblocks_total, int dq_blocksize) {
    if (nblocks_total <= 0 || dq_blocksize != nf4::kDqBlock) return 0;
    return nf4::dq_chunk_count(nblocks_total) * (int64_t)sizeof(double);
}

nf4_status nf4_double_quantize_sharded(const float *absmax, int64_t nblocks, int dq_blocksize,
                                       const double *run_sums_all, int64_t nblocks_total, uint8_t *absmax_q,
                                       float *absmax2, float *offset, void *workspace, int64_t workspace_bytes,
                                       void *stream) {
    if (dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
    if (nblocks < 0 || nblocks_total < 1 || nblocks > nblocks_total) return NF4_ERR_INVALID;
    if (!run_sums_all || !offset || !workspace) return NF4_ERR_INVALID;
    if (nblocks > 0 && (!absmax || !absmax_q || !absmax2)) return NF4_ERR_INVALID;
    if (!aligned16(absmax) || !aligned16(absmax_q) || !aligned16(absmax2) || !aligned16(offset) ||
        !aligned16(workspace) || !aligned16(run_sums_all))
        return NF4_ERR_INVALID;
    if (nf4::dq_chunk_count(nblocks_total) > nf4::dq_max_chunks()) return NF4_ERR_UNSUPPORTED;
    if (workspace_bytes < nf4_double_quantize_sharded_workspace_size(nblocks_total, dq_blocksize))
        return NF4_ERR_INVALID;
    cudaError_t st;
    int sms = sm_count(&st);
    if (st != cudaSuccess) return cuda_status(st);
    return cuda_status(nf4::launch_dq_from_run_sums(absmax, nblocks, run_sums_all, nblocks_total, absmax_q, absmax2,
                                                    offset, static_cast<double *>(workspace), (cudaStream_t)stream,
                                                    sms));
}

nf4_status nf4_dequantize(const uint8_t *packed, const uint8_t *absmax_q, const float *absmax2, const float *offset,
                          int64_t n, int blocksize, int dq_blocksize, void *out, nf4_dtype out_dtype, void *stream) {
    if (blocksize != nf4::kBlock || dq_blocksize != nf4::kDqBlock) return NF4_ERR_UNSUPPORTED;
    if (n < 0 || (n & 1) || (out_dtype != NF4_F32 && out_dtype != NF4_BF16)) return NF4_ERR_INVALID;
    if (n == 0) return NF4_OK;
    if (!packed || !absmax2 || !out) return NF4_ERR_INVALID;
    if (absmax_q == nullptr && offset != nullptr) return NF4_ERR_INVALID;
    if (!aligned16(packed) || !aligned16(absmax_q) || !aligned16(absmax2) || !aligned16(offset) || !aligned16(out))
        return NF4_ERR_INVALID;
    cudaError_t st;
    int sms = sm_count(&st);
    if (st != cudaSuccess) return cuda_status(st);
    return cuda_status(nf4::launch_dequantize(packed, absmax_q, absmax2, offset, n, out, out_dtype == NF4_BF16,
                                              (cudaStream_t)stream, sms));
}

int64_t nf4_lora_linear_workspace_size(int64_t M, int r) {
    if (M <= 0 || r < 0) return 0;
    return nf4::linear_workspace_bytes(M, r);
}

nf4_status nf4_lora_linear_fwd(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed,
                               const uint8_t *absmax_q, const float *absmax2, const float *offset, const void *A,
                               const void *B, int r, float scaling, void *y, void *workspace,
                               int64_t workspace_bytes, void *stream) {
    if (M < 1 || N < 1 || K < nf4::kBlock || (K % nf4::kBlock) != 0) return NF4_ERR_INVALID;
    if (r != 0 && r != 16 && r != 32 && r != 64) return NF4_ERR_UNSUPPORTED;
    if (!x || !packed || !absmax2 || !y) return NF4_ERR_INVALID;
    if (absmax_q == nullptr && offset != nullptr) return NF4_ERR_INVALID;
    const bool lora = (r > 0 && A != nullptr && B != nullptr);
    if (!aligned16(x) || !aligned16(packed) || !aligned16(absmax_q) || !aligned16(absmax2) || !aligned16(offset) ||
        !aligned16(y) || !aligned16(A) || !aligned16(B) || !aligned16(workspace))
        return NF4_ERR_INVALID;
    if (lora && (workspace == nullptr || workspace_bytes < nf4::lora_workspace_bytes(M, r))) return NF4_ERR_INVALID;
    if ((N % 8) != 0) return NF4_ERR_UNSUPPORTED;  // y rows must stay 16-byte aligned
    cudaError_t st;
    int sms = sm_count(&st);
    if (st != cudaSuccess) return cuda_status(st);
    unsigned *err = nf4::device_error_word(&st);
    if (st != cudaSuccess) return cuda_status(st);
    return cuda_status(nf4::launch_lora_linear(x, M, K, N, packed, absmax_q, absmax2, offset, lora ? A : nullptr,
                                               lora ? B : nullptr, lora ? r : 0, scaling, y, workspace,
                                               workspace == nullptr ? 0 : workspace_bytes, (cudaStream_t)stream,
                                               sms, err));
}

int64_t nf4_lora_linear_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int r) {
    if (M < 0 || N < 0 || K < 0 || r <= 0) return 0;
    return nf4::lora_bwd_workspace_bytes(M, N, K, r);
}

nf4_status nf4_lora_linear_bwd(const void *g, const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed,
                               const uint8_t *absmax_q, const float *absmax2, const float *offset, const void *A,
                               const void *B, int r, float scaling, void *dx, float *dA, float *dB, void *workspace,
                               int64_t workspace_bytes, void *stream) {
    if (M < 1 || N < 1 || K < nf4::kBlock || (K % nf4::kBlock) != 0) return NF4_ERR_INVALID;
    if ((N % 8) != 0) return NF4_ERR_UNSUPPORTED;
    if (r != 0 && r != 16 && r != 32 && r != 64) return NF4_ERR_UNSUPPORTED;
    if (!g) return NF4_ERR_INVALID;
    const bool lora = r > 0 && A != nullptr && B != nullptr;
    if (!lora && (dA || dB)) return NF4_ERR_INVALID;
    if ((dA || dB) && !x) return NF4_ERR_INVALID;
    if (dx && (!packed || !absmax2)) return NF4_ERR_INVALID;
    if (absmax_q == nullptr && offset != nullptr) return NF4_ERR_INVALID;
    if (!aligned16(g) || !aligned16(x) || !aligned16(packed) || !aligned16(absmax_q) || !aligned16(absmax2) ||
        !aligned16(offset) || !aligned16(A) || !aligned16(B) || !aligned16(dx) || !aligned16(dA) || !aligned16(dB))
        return NF4_ERR_INVALID;
    const int rr = lora ? r : 0;
    if (lora) {
        if (workspace == nullptr || ((uintptr_t)workspace & 255u) != 0) return NF4_ERR_INVALID;
        if (workspace_bytes < nf4_lora_linear_bwd_workspace_size(M, N, K, r)) return NF4_ERR_INVALID;
    }
    cudaError_t st;
    unsigned *err = nf4::device_error_word(&st);
    if (st != cudaSuccess) return cuda_status(st);
    const int sms = sm_count(&st);
    if (st != cudaSuccess) return cuda_status(st);
    return cuda_status(nf4::launch_lora_linear_bwd(g, x, M, K, N, packed, absmax_q, absmax2, offset,
                                                   lora ? A : nullptr, lora ? B : nullptr, rr, scaling, dx, dA, dB,
                                                   workspace, err, (cudaStream_t)stream, sms));
}

nf4_status nf4_merge_requantize(const uint8_t *packed, const uint8_t *absmax_q, const float *absmax2,
                                const float *offset, int64_t N, int64_t K, const void *A, const void *B, int r,
                                float scaling, uint8_t *packed_out, float *absmax_out, void *stream) {
    if (N < 1 || K < nf4::kBlock || (K % nf4::kBlock) != 0) return NF4_ERR_INVALID;
    if (r < 0) return NF4_ERR_INVALID;
    if (r > nf4::merge_max_rank()) return NF4_ERR_UNSUPPORTED;
    if (!packed || !absmax2 || !packed_out || !absmax_out) return NF4_ERR_INVALID;
    if (absmax_q == nullptr && offset != nullptr) return NF4_ERR_INVALID;
    const bool lora = r > 0 && A != nullptr && B != nullptr;
    if (!aligned16(packed) || !aligned16(absmax_q) || !aligned16(absmax2) || !aligned16(offset) ||
        !aligned16(A) || !aligned16(B) || !aligned16(packed_out) || !aligned16(absmax_out))
        return NF4_ERR_INVALID;
    return cuda_status(nf4::launch_merge_requantize(packed, absmax_q, absmax2, offset, N, K, lora ? A : nullptr,
                                                    lora ? B : nullptr, lora ? r : 0, scaling, packed_out,
                                                    absmax_out, (cudaStream_t)stream));
}

nf4_status nf4_selftest_wait_timeout(int64_t limit_ns, void *stream) {
    if (limit_ns < 1 || limit_ns > 1000000000) return NF4_ERR_INVALID;
    return cuda_status(nf4::launch_selftest_wait((unsigned long long)limit_ns, (cudaStream_t)stream));
}

nf4_status nf4_device_status(void *stream) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_status(e);
    unsigned *err = nf4::device_error_word(&e);
    if (e != cudaSuccess) return cuda_status(e);
    unsigned host = 0;
    e = cudaMemcpy(&host, err, sizeof host, cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_status(e);
    if (host != 0) {
        unsigned zero = 0;
        e = cudaMemcpy(err, &zero, sizeof zero, cudaMemcpyHostToDevice);
        if (e != cudaSuccess) return cuda_status(e);
        return NF4_ERR_TIMEOUT;
    }
    return NF4_OK;
}

}  // extern "C"
