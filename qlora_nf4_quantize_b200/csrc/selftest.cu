// selftest.cu -- exercises the bounded-wait expiry path on the GPU without a
// fault: one thread runs the kernels' own bounded wait (mbar_wait) on an
// mbarrier that nothing arrives on, with the caller's limit instead of the
// default second; it gives up, raises the device error word and returns, the
// path every fused kernel takes when one of its waits expires.  The pages
// have no counterpart; this is the library's failure-detection check.
#include "mbarrier.cuh"

namespace nf4 {

unsigned *device_error_word(cudaError_t *status);

namespace {

__global__ void k_selftest_wait(unsigned long long limit_ns, unsigned *err) {
    __shared__ uint64_t bar;
    __shared__ int abort;
    if (threadIdx.x != 0) return;
    abort = 0;
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    // the kernels' own bounded wait (mbarrier.cuh), on a phase that never
    // completes: it gives up after limit_ns, raises the abort flag and the
    // device error word, and returns false
    mbar_wait(&bar, 0, &abort, err, limit_ns);
}

}  // namespace

cudaError_t launch_selftest_wait(unsigned long long limit_ns, cudaStream_t stream) {
    cudaError_t e = cudaSuccess;
    unsigned *err = device_error_word(&e);
    if (e != cudaSuccess) return e;
    k_selftest_wait<<<1, 32, 0, stream>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace nf4
