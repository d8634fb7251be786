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
// Division-free exact code selection: instead of the per-element IEEE
// division, each element uses q = RN(w * rc), rc the reciprocal of c1 to
// within 1 ulp, which is within 2^-22 of x = RN(w / c1).  A 129-cell table
// indexed by round(64 q) gives the code below the cell and the (at most one)
// threshold inside the cell widened by 2^-18; code = base + (q > t).  When |q - t| <= 2^-18 the decision could
// differ from the exact one and the element falls back to __fdiv_rn and a
// full threshold count.  Each table word stores the threshold's bits with the
// low 4 mantissa bits replaced by the base code (a perturbation below 2^-20,
// covered by the 2^-18 margin).
#include "nf4_device.cuh"

namespace nf4 {
namespace {

constexpr float kAmbiguity = 0x1p-18f;
constexpr int kCells = 129;       // cells 0..128 cover q in [-1, 1]
constexpr int kCellTable = 256;   // indexed by the low byte of RN(64 q) + 64 (+ 1.5 * 2^23)
constexpr int kQuantThreads = 256;
#ifndef NF4_QUANT_RCP_APPROX
#define NF4_QUANT_RCP_APPROX 1
#endif
// CTAs per SM in the grid; 0 = the number resident at once (occupancy query)
#ifndef NF4_QUANT_CTAS_PER_SM
#define NF4_QUANT_CTAS_PER_SM 0
#endif

__device__ __forceinline__ int exact_code(float w, float c1, const float *s_t) {
    return code_of_quotient(__fdiv_rn(w, c1), s_t);
}

// Fill the thresholds and the cell table in shared memory (once per CTA).
__device__ void build_tables(float *s_t, uint32_t *s_cell) {
    int tid = threadIdx.x;
    fill_thresholds(s_t);
    __syncthreads();
    if (tid >= kCells && tid < kCellTable) s_cell[tid] = 0x40800000u | 15u;  // never reached by finite q
    if (tid < kCells) {
        // cell tid holds q with RN(64 q) = tid - 64, i.e. q in [lo, hi]
        float lo = ((float)tid - 64.5f) * 0.015625f;
        float hi = ((float)tid - 63.5f) * 0.015625f;
        int base = 0;
        uint32_t word = 0x40800000u;  // 4.0f: no threshold near this cell
        for (int i = 0; i < 15; ++i) {
            float t = s_t[i];
            if (t < lo - kAmbiguity) ++base;
            else if (t <= hi + kAmbiguity) word = __float_as_uint(t);
        }
        s_cell[tid] = (word & ~15u) | (uint32_t)base;
    }
    __syncthreads();
}

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

    uint32_t word;  // byte j = code[2j] << 4 | code[2j+1], bytes 0..3
    if (c1 == 0.0f) {
        word = 0x77777777u;
    } else {
        bool amb = true;  // take the exact path
        word = 0;
        if (c1 >= 0x1p-125f && c1 < 0x1p125f) {
            // (outside this range 1/c1 may overflow or be subnormal, so the
            // 2^-22 error bound of the fast path would not hold)
#if NF4_QUANT_RCP_APPROX
            // hardware reciprocal, at most 1 ulp from 1 / c1 (PTX rcp.approx):
            // |q - x| stays below 2^-22 (2^-23 + 2 half-ulps of rounding for
            // |w / c1| <= 1), the bound the 2^-18 margin covers
            float rc;
            asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(rc) : "f"(c1));
#else
            const float rc = __frcp_rn(c1);
#endif
            uint64_t rc2, k64, kmagic;
            asm("mov.b64 %0, {%1, %1};" : "=l"(rc2) : "f"(rc));
            asm("mov.b64 %0, {%1, %1};" : "=l"(k64) : "f"(64.0f));
            asm("mov.b64 %0, {%1, %1};" : "=l"(kmagic) : "f"(12582976.0f));  // 1.5 * 2^23 + 64
            float dmin = 1.0f;  // smallest |q - t| of the group
            // pairs (6, 7), (4, 5), (2, 3), (0, 1): codes enter the word most
            // significant nibble first (byte m = code[2m] << 4 | code[2m+1])
#pragma unroll
            for (int i = 6; i >= 0; i -= 2) {
                // q = RN(w * rc) and RN(64 q) + 64 in the low bits of
                // f = RN(64 q + 1.5 * 2^23 + 64), two elements per packed op
                uint64_t vv, qq, ff;
                asm("mov.b64 %0, {%1, %2};" : "=l"(vv) : "f"(v[i]), "f"(v[i + 1]));
                asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(qq) : "l"(vv), "l"(rc2));
                asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(ff) : "l"(qq), "l"(k64), "l"(kmagic));
                float q[2], f[2];
                asm("mov.b64 {%0, %1}, %2;" : "=f"(q[0]), "=f"(q[1]) : "l"(qq));
                asm("mov.b64 {%0, %1}, %2;" : "=f"(f[0]), "=f"(f[1]) : "l"(ff));
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    // RN(64 q) + 64 is in [0, 128] for finite inputs; the byte
                    // mask keeps any input inside the 256-entry table
                    const uint32_t e = s_cell[__float_as_uint(f[j]) & 0xFFu];
                    const float t = __uint_as_float(e);
                    const uint32_t code = (e & 15u) + ((q[j] > t) ? 1u : 0u);
                    word = (word << 4) | code;
                    dmin = fminf(dmin, fabsf(q[j] - t));
                }
            }
            amb = dmin <= kAmbiguity;  // rare: some quotient is within 2^-18 of a threshold
        }
        if (amb) {
            word = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                word += (uint32_t)exact_code(v[i], c1, s_t) << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
        }
    }
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
    build_tables(s_t, s_cell);

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
