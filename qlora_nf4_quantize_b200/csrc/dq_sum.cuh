// dq_sum.cuh -- the binary64 sum of one run of first-level constants, as the
// double quantization's centring mean defines it ("QLoRA: Mathematical
// Foundations ...", section "Double Quantization (DQ)": the per-tensor mean;
// READING: each run of 256 constants summed sequentially in index order),
// computed by one warp.
//
// The sequential fp64 sum of a run equals its exact sum whenever every
// partial sum is representable.  The constants are >= 0 and multiples of
// 2^(emin - 150) (emin = smallest biased exponent among the non-zero ones, 1
// for subnormals), and the total is below 256 * 2^(emax - 126); if
// emax - emin <= 21 every subset sum is exact in fp64, so any summation order
// gives the sequential result.  Otherwise lane 0 sums the run sequentially.
#pragma once

#include "nf4_device.cuh"

namespace nf4 {

__device__ __forceinline__ int biased_exp(float v) {
    int e = (int)((__float_as_uint(v) >> 23) & 0xFF);
    return e == 0 ? 1 : e;
}

// Sum of c1[0 .. cnt) (cnt <= 256), every lane of the calling warp gets it.
// c1 may point to global or shared memory.
__device__ __forceinline__ double run_sum_fp64(const float *c1, int64_t cnt, int lane) {
    double sum = 0.0;
    int emin = 255, emax = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        int64_t k = lane + 32 * i;
        if (k < cnt) {
            float v = c1[k];
            sum += (double)v;
            if (v != 0.0f) {
                int e = biased_exp(v);
                emin = min(emin, e);
                emax = max(emax, e);
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
        emin = min(emin, __shfl_xor_sync(0xFFFFFFFFu, emin, o));
        emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
    }
    if (emax != 0 && emax - emin > 21) {  // rare: reproduce the sequential order
        double acc = 0.0;
        if (lane == 0)
            for (int64_t k = 0; k < cnt; ++k) acc += (double)c1[k];
        sum = __shfl_sync(0xFFFFFFFFu, acc, 0);
    }
    return sum;
}

}  // namespace nf4
