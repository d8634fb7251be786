// quantize.cu -- K1: blockwise NF4 quantization.
//
// "QLoRA: Mathematical Foundations ..." (llms.blog), section "Block-Wise
// Quantization Mechanics": c1 = max_j |w_j| over each contiguous block of 64,
// code_j = arg-min_i |w_j / c1 - q_i|.  The quotient is the IEEE binary32
// quotient; ties go to the lower index, i.e. code = #{i : x > t_i} with
// t_i = RD_f32((q_i + q_{i+1}) / 2) (the exact midpoint rounded down).
//
// Layout of the work: one thread owns groups of 8 consecutive elements, so
// the 8 lanes l..l+7 (l a multiple of 8) of a warp own one 64-block; c1 is a
// 3-step xor-shuffle max inside that lane group.  Each thread writes its 8
// codes as one 32-bit word (4 packed bytes), a warp 128 contiguous bytes.
//
// The code selection itself (division-free, exact) is encode8 in
// nf4_encode.cuh.
#include "nf4_encode.cuh"

namespace nf4 {
namespace {

constexpr int kQuantThreads = 256;
// CTAs per SM in the grid; 0 = the number resident at once (occupancy query)
#ifndef NF4_QUANT_CTAS_PER_SM
#define NF4_QUANT_CTAS_PER_SM 0
#endif

template <bool kBf16>
__device__ __forceinline__ void load8(const void *w, int64_t e0, int64_t n, float v[8]) {
    if (e0 + 8 <= n) {
        if constexpr (kBf16) {
            uint4 u = __ldg(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(w) + e0));
            uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[2 * i] = __uint_as_float(p[i] << 16);
                v[2 * i + 1] = __uint_as_float(p[i] & 0xFFFF0000u);
            }
        } else {
            const float4 *src = reinterpret_cast<const float4 *>(static_cast<const float *>(w) + e0);
            float4 a = __ldg(src), b = __ldg(src + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int64_t e = e0 + i;
            float x = 0.0f;
            if (e < n) {
                if constexpr (kBf16) {
                    uint16_t h = __ldg(reinterpret_cast<const unsigned short *>(w) + e);
                    x = __uint_as_float((uint32_t)h << 16);
                } else {
                    x = __ldg(static_cast<const float *>(w) + e);
                }
            }
            v[i] = x;
        }
    }
}

// One group = 8 consecutive elements, owned by one thread; the 8 lanes of a
// lane group (lane / 8) own one 64-block.  Consecutive groups of a thread are
// a grid stride apart (a multiple of 8 groups, so lane groups still cover
// whole blocks).
template <bool kBf16>
__device__ __forceinline__ void quantize_group(float v[8], int64_t g, int64_t e0, int64_t n, int lane,
                                               const float *s_t, const uint32_t *s_cell,
                                               uint8_t *__restrict__ packed, float *__restrict__ absmax) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 2));
    a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, 4));
    const float c1 = a;
    if (e0 >= n) return;
    if ((lane & 7) == 0) absmax[g >> 3] = c1;

    const uint32_t word = encode8(v, c1, s_t, s_cell);  // byte j = code[2j] << 4 | code[2j+1]
    if (e0 + 8 <= n) {
        reinterpret_cast<uint32_t *>(packed)[g] = word;
    } else {
        for (int j = 0; 2 * j < (int)(n - e0); ++j) packed[(e0 >> 1) + j] = (uint8_t)(word >> (8 * j));
    }
}

template <bool kBf16>
__global__ void __launch_bounds__(kQuantThreads) k_quantize(const void *__restrict__ w, int64_t n,
                                                             uint8_t *__restrict__ packed,
                                                             float *__restrict__ absmax) {
    __shared__ float s_t[16];
    __shared__ uint32_t s_cell[kCellTable];
    pdl_wait_then_release();
    build_code_tables(s_t, s_cell);

    const int lane = threadIdx.x & 31;
    const int64_t ngroups = (n + 7) >> 3;
    const int64_t stride = (int64_t)gridDim.x * kQuantThreads;
    // the trip count depends only on blockIdx, so whole warps stay converged
    for (int64_t base = (int64_t)blockIdx.x * kQuantThreads; base < ngroups; base += stride) {
        const int64_t g = base + threadIdx.x;
        float v[8];
        load8<kBf16>(w, g << 3, n, v);
        quantize_group<kBf16>(v, g, g << 3, n, lane, s_t, s_cell, packed, absmax);
    }
}

}  // namespace

cudaError_t launch_quantize(const void *w, bool bf16, int64_t n, uint8_t *packed, float *absmax,
                            cudaStream_t stream, int num_sms) {
    if (n == 0) return cudaSuccess;
    int64_t ngroups = (n + 7) / 8;
    int64_t span = (int64_t)kQuantThreads;
    int64_t want = (ngroups + span - 1) / span;
    // one wave: as many CTAs as are resident at once (registers bound it to
    // 5 per SM), so that no SM idles while a second, partial wave finishes
    int per_sm = NF4_QUANT_CTAS_PER_SM;
    if (per_sm <= 0) {
        cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
            &per_sm, bf16 ? k_quantize<true> : k_quantize<false>, kQuantThreads, 0);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) per_sm = 1;
    }
    int64_t cap = (int64_t)num_sms * per_sm;
    int grid = (int)(want < cap ? want : cap);
    if (bf16) return launch_pdl(k_quantize<true>, dim3(grid), dim3(kQuantThreads), 0, stream, 1, w, n, packed, absmax);
    return launch_pdl(k_quantize<false>, dim3(grid), dim3(kQuantThreads), 0, stream, 1, w, n, packed, absmax);
}

}  // namespace nf4
