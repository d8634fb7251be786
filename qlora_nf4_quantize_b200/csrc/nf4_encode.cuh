// nf4_encode.cuh -- NF4 code selection for a group of 8 elements of one
// 64-block, shared by the quantizer (quantize.cu) and the merge-and-requantize
// kernel (merge.cu).
//
// "QLoRA: Mathematical Foundations ..." (llms.blog), section "Block-Wise
// Quantization Mechanics": code_j = arg-min_i |w_j / c1 - q_i| with the IEEE
// binary32 quotient; ties go to the lower index, i.e. code = #{i : x > t_i},
// t_i = RD_f32((q_i + q_{i+1}) / 2) (the exact midpoint rounded down).
//
// Division-free exact selection: instead of the per-element IEEE division,
// each element uses q = RN(w * rc), rc the reciprocal of c1 to within 1 ulp,
// which is within 2^-22 of x = RN(w / c1).  A 129-cell table indexed by
// round(64 q) gives the code below the cell and the (at most one) threshold
// inside the cell widened by 2^-18; code = base + (q > t).  When |q - t| <=
// 2^-18 the decision could differ from the exact one and the group falls back
// to __fdiv_rn and a full threshold count.  Each table word stores the
// threshold's bits with the low 4 mantissa bits replaced by the base code (a
// perturbation below 2^-20, covered by the 2^-18 margin).
#pragma once

#include "nf4_device.cuh"

namespace nf4 {

constexpr float kAmbiguity = 0x1p-18f;
constexpr int kCells = 129;      // cells 0..128 cover q in [-1, 1]
constexpr int kCellTable = 256;  // indexed by the low byte of RN(64 q) + 64 (+ 1.5 * 2^23)

// 1: the compare q > t is taken from the sign of t - q, the difference the
// ambiguity test needs anyway
#ifndef NF4_ENCODE_SIGN
#define NF4_ENCODE_SIGN 1
#endif

#ifndef NF4_QUANT_RCP_APPROX
#define NF4_QUANT_RCP_APPROX 1
#endif

// Fill the thresholds (s_t[15]) and the cell table (s_cell[256]) in shared
// memory; every thread of the CTA calls it (it synchronises the CTA).
__device__ __forceinline__ void build_code_tables(float *s_t, uint32_t *s_cell) {
    const int tid = threadIdx.x;
    fill_thresholds(s_t);
    __syncthreads();
    for (int c = tid; c < kCellTable; c += blockDim.x) {
        if (c >= kCells) {
            s_cell[c] = 0x40800000u | 15u;  // never reached by finite q
            continue;
        }
        // cell c holds q with RN(64 q) = c - 64, i.e. q in [lo, hi]
        const float lo = ((float)c - 64.5f) * 0.015625f;
        const float hi = ((float)c - 63.5f) * 0.015625f;
        int base = 0;
        uint32_t word = 0x40800000u;  // 4.0f: no threshold near this cell
        for (int i = 0; i < 15; ++i) {
            const float t = s_t[i];
            if (t < lo - kAmbiguity) ++base;
            else if (t <= hi + kAmbiguity) word = __float_as_uint(t);
        }
        s_cell[c] = (word & ~15u) | (uint32_t)base;
    }
    __syncthreads();
}

// The 8 codes of elements v[0..7] of a block with constant c1 (>= 0, the
// block's absmax) as one packed word: byte m = code[2m] << 4 | code[2m+1].
__device__ __forceinline__ uint32_t encode8(const float v[8], float c1, const float *s_t, const uint32_t *s_cell) {
    if (c1 == 0.0f) return 0x77777777u;
    uint32_t word = 0;
    bool amb = true;  // take the exact path
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
        // significant nibble first
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
#if NF4_ENCODE_SIGN
                // d = RN(t - q) is negative exactly when q > t (a nonzero
                // difference of two finite binary32 values in [-4, 4] never
                // rounds to zero, and t - t = +0): its sign bit is the compare
                const float d = t - q[j];
                word = (word << 4) + (e & 15u) + (__float_as_uint(d) >> 31);
                dmin = fminf(dmin, fabsf(d));
#else
                const uint32_t code = (e & 15u) + ((q[j] > t) ? 1u : 0u);
                word = (word << 4) | code;
                dmin = fminf(dmin, fabsf(q[j] - t));
#endif
            }
        }
        amb = dmin <= kAmbiguity;  // rare: some quotient is within 2^-18 of a threshold
    }
    if (amb) {
        word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i)
            word += (uint32_t)code_of_quotient(__fdiv_rn(v[i], c1), s_t) << (8 * (i >> 1) + ((i & 1) ? 0 : 4));
    }
    return word;
}

}  // namespace nf4
