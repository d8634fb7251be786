// mma_util.cuh -- warp-level bf16 MMA and the NF4 register lookup table.
#pragma once

#include "nf4_device.cuh"

namespace nf4 {

// D = A * B + D for one m16n8k16 bf16 tile with fp32 accumulators.
// a: 4 registers (bf16x2) of the 16x16 row-major A fragment, b: 2 registers
// of the 16x8 column-major B fragment, d: 4 fp32 accumulators.
__device__ __forceinline__ void mma_bf16_16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Per-block lookup table of the 16 dequantized bf16 weights
//   e_i = RNE_bf16( RN_f32( q_i * c ) ),  i = 0..15,
// held as byte planes: L0..L3 carry the low bytes of e_0..e_15 (four per
// register), H0..H3 the high bytes.  Built once per 64-block from its
// reconstructed constant c (16 binary32 multiplies, 8 bf16x2 conversions,
// 8 byte permutes).
struct Lut {
    uint32_t L0, L1, L2, L3, H0, H1, H2, H3;
};

__device__ __forceinline__ Lut make_lut(float c) {
    // P[j] = (RNE_bf16(RN(q[2j] c)), RNE_bf16(RN(q[2j+1] c))): the two
    // products are one packed f32x2 multiply (each half rounded to nearest,
    // as two binary32 multiplies)
    uint64_t cc;
    asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
    uint32_t P[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        uint64_t qq, d;
        asm("mov.b64 %0, {%1, %2};" : "=l"(qq) : "f"(c_levels[2 * j]), "f"(c_levels[2 * j + 1]));
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(qq), "l"(cc));
        float lo, hi;
        asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
        P[j] = pack_bf16x2(lo, hi);
    }
    Lut t;
    t.L0 = __byte_perm(P[0], P[1], 0x6420); t.H0 = __byte_perm(P[0], P[1], 0x7531);
    t.L1 = __byte_perm(P[2], P[3], 0x6420); t.H1 = __byte_perm(P[2], P[3], 0x7531);
    t.L2 = __byte_perm(P[4], P[5], 0x6420); t.H2 = __byte_perm(P[4], P[5], 0x7531);
    t.L3 = __byte_perm(P[6], P[7], 0x6420); t.H3 = __byte_perm(P[6], P[7], 0x7531);
    return t;
}

// Look up four codes held in the low 16 bits of p16 (two packed bytes:
// byte 0 = e0 << 4 | e1, byte 1 = e2 << 4 | e3, so the nibbles from bit 0 up
// are e1, e0, e3, e2).  Returns the bf16 weights as two bf16x2 words:
// lo01 = (e0 in the low half, e1 in the high half), lo23 = (e2, e3).
// Each byte permute selects within 8 bytes, so codes 0-7 and 8-15 are looked
// up separately and merged on bit 3 of each code.
__device__ __forceinline__ void lut_lookup4_sel(const Lut &t, uint32_t s, uint32_t s2, uint32_t &w01,
                                                uint32_t &w23) {
    const uint32_t loA = __byte_perm(t.L0, t.L1, s), loB = __byte_perm(t.L2, t.L3, s);
    const uint32_t hiA = __byte_perm(t.H0, t.H1, s), hiB = __byte_perm(t.H2, t.H3, s);
    const uint32_t lo = __byte_perm(loA, loB, s2), hi = __byte_perm(hiA, hiB, s2);
    w01 = __byte_perm(lo, hi, 0x4051);
    w23 = __byte_perm(lo, hi, 0x6273);
}

static __constant__ uint32_t c_selector_mul[2] = {1u << 16, 1u << 31};

// Selectors of the byte permutes for the 8 codes of one 32-bit word of packed
// codes: s = low 3 bits of each code (bit 3 cleared, so no sign-replicate
// mode), s2 = per output byte i, i + 4 * (bit 3 of code i).  A byte permute
// reads only the low 16 bits of its selector, so the high halves serve the
// codes of bytes 2 and 3 after a 16-bit shift.
__device__ __forceinline__ void lut_selectors(uint32_t w, uint32_t &s_lo, uint32_t &s_hi, uint32_t &s2_lo,
                                              uint32_t &s2_hi) {
    // The right shifts are high halves of products (w >> k = umulhi(w, 2^(32-k))),
    // which issue on the multiply-add pipe and leave the integer pipe, the
    // bottleneck of the dequantization, to the masks and byte permutes.
    // The multipliers are read from constant memory so that the compiler
    // does not turn the products back into shifts.
    const uint32_t m16 = c_selector_mul[0], m31 = c_selector_mul[1];
    s_lo = w & 0x77777777u;
    s_hi = __umulhi(s_lo, m16);
    s2_lo = (__umulhi(w, m31) & 0x44444444u) | 0x32103210u;
    s2_hi = __umulhi(s2_lo, m16);
}

__device__ __forceinline__ void lut_lookup4(const Lut &t, uint32_t p16, uint32_t &w01, uint32_t &w23) {
    lut_lookup4_sel(t, p16 & 0x7777u, ((p16 >> 1) & 0x4444u) | 0x3210u, w01, w23);
}

// The 8 weights of one 32-bit word of packed codes (bytes 0..3, two codes
// each) as four bf16x2 words, in element order.
__device__ __forceinline__ void lut_lookup8(const Lut &t, uint32_t w, uint32_t out[4]) {
    uint32_t s_lo, s_hi, s2_lo, s2_hi;
    lut_selectors(w, s_lo, s_hi, s2_lo, s2_hi);
    lut_lookup4_sel(t, s_lo, s2_lo, out[0], out[1]);
    lut_lookup4_sel(t, s_hi, s2_hi, out[2], out[3]);
}

}  // namespace nf4

namespace nf4 {

// Shared-memory table of unscaled level pairs for byte-wise dequantization:
// entry b (one packed byte: code of element 2j in the high nibble, 2j+1 in
// the low nibble) = (q[b >> 4], q[b & 15]).  kPairCopies interleaved copies,
// entry b of copy c at float2 index 16 b + c, so the 16 lanes of a half-warp
// (which a 64-bit shared load serves together) read 16 different bank pairs
// whatever bytes they look up.  32 KB.
constexpr int kPairCopies = 16;
constexpr int kPairTableFloat2 = 256 * kPairCopies;

__device__ __forceinline__ void fill_pair_table(float2 *tbl) {
    for (int i = threadIdx.x; i < kPairTableFloat2; i += blockDim.x) {
        const int b = i / kPairCopies;
        tbl[i] = make_float2(c_levels[b >> 4], c_levels[b & 15]);
    }
}

// Two bf16 weights of one packed byte: RNE_bf16(RN_f32(q * c)) for both
// nibbles, returned as a bf16x2 word (element 2j in the low half).
// tbl_lane = table + (lane & 15).
// The two products are one packed f32x2 multiply (each lane rounded to
// nearest, as two binary32 multiplies).
__device__ __forceinline__ uint32_t pair_lookup(const float2 *tbl_lane, uint32_t byte, float c) {
    const float2 q = tbl_lane[byte * kPairCopies];
    uint64_t qq, cc, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(qq) : "f"(q.x), "f"(q.y));
    asm("mov.b64 %0, {%1, %1};" : "=l"(cc) : "f"(c));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(qq), "l"(cc));
    float lo, hi;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(d));
    return pack_bf16x2(lo, hi);
}

// Same four-code lookup as lut_lookup4 (same output layout) through the
// shared-memory pair table: p16 holds two packed bytes in its low 16 bits.
__device__ __forceinline__ void pair_lookup4(const float2 *tbl_lane, uint32_t p16, float c, uint32_t &w01,
                                             uint32_t &w23) {
    w01 = pair_lookup(tbl_lane, __byte_perm(p16, 0u, 0x4440), c);
    w23 = pair_lookup(tbl_lane, __byte_perm(p16, 0u, 0x4441), c);
}

// pair_lookup4 with the table addressed by a 32-bit shared-memory address
// (base_lane = shared address of table + (lane & 15)) and c given as the
// packed pair (c, c): per byte one byte permute, one multiply-add for the
// address, one 64-bit shared load, one packed f32x2 multiply (each half
// rounded to nearest) and one conversion to bf16x2.
__device__ __forceinline__ void pair_lookup4_s(uint32_t base_lane, uint32_t p16, uint64_t cc, uint32_t &w01,
                                               uint32_t &w23) {
    asm("{\n\t"
        ".reg .b32 b0, b1, l0, h0, l1, h1;\n\t"
        ".reg .b64 q0, q1;\n\t"
        "prmt.b32 b0, %2, 0, 0x4440;\n\t"
        "prmt.b32 b1, %2, 0, 0x4441;\n\t"
        "mad.lo.u32 b0, b0, %5, %3;\n\t"
        "mad.lo.u32 b1, b1, %5, %3;\n\t"
        "ld.shared.b64 q0, [b0];\n\t"
        "ld.shared.b64 q1, [b1];\n\t"
        "mul.rn.f32x2 q0, q0, %4;\n\t"
        "mul.rn.f32x2 q1, q1, %4;\n\t"
        "mov.b64 {l0, h0}, q0;\n\t"
        "mov.b64 {l1, h1}, q1;\n\t"
        "cvt.rn.bf16x2.f32 %0, h0, l0;\n\t"
        "cvt.rn.bf16x2.f32 %1, h1, l1;\n\t"
        "}"
        : "=r"(w01), "=r"(w23)
        : "r"(p16), "r"(base_lane), "l"(cc), "n"(kPairCopies * 8));
}

__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}

}  // namespace nf4
