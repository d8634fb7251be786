// selftest.cu -- exercises the bounded-wait expiry path on the GPU without a
// fault: one thread waits on an mbarrier that nothing arrives on, gives up
// after the caller's limit, raises the device error word and returns, exactly
// as the fused kernels do when a wait expires.  The pages have no counterpart;
// this is the library's failure-detection check.
#include "mbarrier.cuh"

namespace nf4 {

unsigned *device_error_word(cudaError_t *status);

namespace {

__global__ void k_selftest_wait(unsigned long long limit_ns, unsigned *err) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait_sleep(&bar, 0)) {  // phase 0 never completes
        if (global_ns() - t0 > limit_ns) {
            atomicOr(err, 1u);
            return;
        }
    }
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
