// decode.cu -- K4: fused NF4-dequantizing linear for decode-size token counts
// (M <= 16), y = x W~^T + [t_hi | t_lo] [B | B]^T.
//
// "QLoRA: Mathematical Foundations ...", section "Forward Pass Computation":
// the weight is dequantized on the fly into registers and never written to
// memory; compute dtype bf16 with fp32 accumulation.  The W~ values are
// exactly the bf16 outputs of nf4_dequantize (RNE_bf16(RN_f32(q * c1'))).
//
// The call streams the packed weight once (0.5 B + 1/64 B per parameter);
// the kernel is built so that the per-weight work stays close to the time of
// that stream and the stream never waits on it:
//   - one CTA of 16 warps per SM owns a contiguous range of 16-row weight
//     tiles.  The tokens form kNT MMA column tiles of 8 (kNT = 1 up to 8
//     tokens, 2 up to 16).  A unit is (tile, slice of 256 / kNT columns):
//     16 rows x 128 / kNT bytes of codes, so that a warp's x fragments
//     (kNT tiles x 256 / kNT columns) take the same 32 registers for either
//     kNT.  With S <= 16 slices per row, warp w takes slice w % S of the
//     tiles w / S, w / S + 16 / S, ..., so its x fragments stay in registers
//     for the whole call; with S > 16 warp w takes slices w, w + 16, ... and
//     runs a chunk of tiles (below) slice by slice -- every tile of the
//     chunk at slice w, then at w + 16, ... -- loading x once per slice.
//   - each warp streams its own units into its own ring of 3 unit slots in
//     shared memory with asynchronous 16-byte copies (cp.async, zero-filled
//     outside the weight; 128-byte rows have their 16-byte chunks
//     XOR-swizzled by row so that the fragment reads are conflict-free,
//     64-byte rows need no swizzle), three units ahead of the one it
//     multiplies.  No warp waits for another until the end of a chunk.
//   - the MMA is the warp-level m16n8k16 with the weight as the A operand.
//     Within a slice the K index is permuted so that lane t of a quad holds,
//     at MMA step j, elements 4j..4j+3 of its 64 / kNT contiguous columns
//     of the slice (rows g and g + 8): 64-block t for kNT = 1, half of
//     64-block t / 2 for kNT = 2.  x uses the same permutation (one 8-byte
//     fragment per step and token tile).  A lane's columns therefore lie in
//     one 64-block: one constant per row and unit.  With one token tile
//     even and odd steps accumulate into separate chains.
//   - dequantization through a shared-memory table of unscaled level pairs
//     (q[b >> 4], q[b & 15]) for every code byte b, in 16 copies so that the
//     16 lanes a 64-bit shared load serves together never share a bank; the
//     entry of a byte is addressed by one byte permute (the table starts on
//     a 64 KB boundary of the shared window with entries 256 bytes apart, so
//     byte b becomes bits 8..15 of the address), then one packed f32x2
//     multiply by (c, c) and one bf16x2 conversion: four instructions per
//     two weights.  (The per-block register table of mma_util.cuh, looked
//     up by byte permutes, costs more integer-pipe issue than the table's
//     shared-memory reads; mixing the two was slower.)
//   - block constants are loaded two units ahead into registers.
//   - each warp writes the partial 16 x 8 kNT tile of each unit to shared
//     memory (slot = slice, or warp when S > 16); once a chunk of tiles is
//     done the CTA adds the slots in slot order (so the result does not
//     depend on timing), adds the LoRA K-extension (2r columns, A = [B | B],
//     B operand = [t_hi | t_lo]) by MMA and stores.
// The kernel has no spin-waits: copies are tracked per thread (cp.async
// groups) and the warps meet only at CTA barriers.
#include "decode_split.h"
#include "mma_util.cuh"

namespace nf4 {
namespace {

constexpr int kDThreads = kDWarps * 32;

// Unit geometry for kNT token tiles of 8.
template <int kNT>
struct DGeom {
    static constexpr uint32_t kRowBytes = 128 / kNT;  // code bytes of a row in a unit
    static constexpr uint32_t kUnitBytes = 16 * kRowBytes;
    static constexpr uint32_t kRingBytes = kDWarps * kDRing * kUnitBytes;
    static constexpr int kWords = 8 / kNT;          // code words of a row per lane
    static constexpr int kBlocksPerUnit = 4 / kNT;  // 64-blocks of a row in a unit
    static constexpr int kXFrags = 16 / kNT;        // 8-byte x fragments per token tile
    static constexpr int kTileFloats = 128 * kNT;   // partial tile: 16 rows x 8 kNT tokens
    // MMA accumulator chains per token tile: even and odd steps apart with
    // one tile; with two, the tiles' chains already alternate
    static constexpr int kChains = kNT == 1 ? 2 : 1;
    static_assert(kRingBytes == decode_ring_bytes(kNT) && kBlocksPerUnit == decode_blocks_per_unit(kNT),
                  "unit geometry of decode_split.h");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

// Four code bytes of one word through the pair table: out[b] = bf16x2 of
// byte b (element of the high nibble in the low half).  base_lane = table
// address | 8 * lane.
__device__ __forceinline__ void pair_word(uint32_t base_lane, uint32_t w, uint64_t cc, uint32_t out[4]) {
    asm volatile(
        "{\n\t"
        ".reg .b32 a0, a1, a2, a3, l0, h0, l1, h1, l2, h2, l3, h3;\n\t"
        ".reg .b64 q0, q1, q2, q3;\n\t"
        "prmt.b32 a0, %4, %5, 0x7604;\n\t"
        "prmt.b32 a1, %4, %5, 0x7614;\n\t"
        "prmt.b32 a2, %4, %5, 0x7624;\n\t"
        "prmt.b32 a3, %4, %5, 0x7634;\n\t"
        "ld.shared.b64 q0, [a0];\n\t"
        "ld.shared.b64 q1, [a1];\n\t"
        "ld.shared.b64 q2, [a2];\n\t"
        "ld.shared.b64 q3, [a3];\n\t"
        "mul.rn.f32x2 q0, q0, %6;\n\t"
        "mul.rn.f32x2 q1, q1, %6;\n\t"
        "mul.rn.f32x2 q2, q2, %6;\n\t"
        "mul.rn.f32x2 q3, q3, %6;\n\t"
        "mov.b64 {l0, h0}, q0;\n\t"
        "mov.b64 {l1, h1}, q1;\n\t"
        "mov.b64 {l2, h2}, q2;\n\t"
        "mov.b64 {l3, h3}, q3;\n\t"
        "cvt.rn.bf16x2.f32 %0, h0, l0;\n\t"
        "cvt.rn.bf16x2.f32 %1, h1, l1;\n\t"
        "cvt.rn.bf16x2.f32 %2, h2, l2;\n\t"
        "cvt.rn.bf16x2.f32 %3, h3, l3;\n\t"
        "}"
        : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
        : "r"(w), "r"(base_lane), "l"(cc));
}

// One unit: 16 / kNT MMA steps per token tile over the lane's columns of
// the two rows (row g: constant c0, row g + 8: c1).
template <int kNT>
__device__ __forceinline__ void mma_unit(const uint32_t (&w)[2][8 / kNT], float c0, float c1, uint32_t base_lane,
                                         const uint2 (&xr)[kNT][16 / kNT],
                                         float (&acc)[kNT][DGeom<kNT>::kChains][4]) {
    constexpr int kOdd = DGeom<kNT>::kChains - 1;  // chain of the odd steps
    const uint64_t cc0 = pack_f32x2(c0, c0), cc1 = pack_f32x2(c1, c1);
#pragma unroll
    for (int q = 0; q < 8 / kNT; ++q) {  // packed word q = MMA steps 2q, 2q+1
        uint32_t wa[4], wb[4];
        pair_word(base_lane, w[0][q], cc0, wa);
        pair_word(base_lane, w[1][q], cc1, wb);
        const uint32_t a0[4] = {wa[0], wb[0], wa[1], wb[1]};
        const uint32_t a1[4] = {wa[2], wb[2], wa[3], wb[3]};
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
            mma_bf16_16816(acc[nt][0], a0, xr[nt][2 * q].x, xr[nt][2 * q].y);
            mma_bf16_16816(acc[nt][kOdd], a1, xr[nt][2 * q + 1].x, xr[nt][2 * q + 1].y);
        }
    }
}

// Shared-memory layout (offsets in the shared window, decode_split.h): the
// pair table at 64 KB (so that byte b of a code word, permuted into bits
// 8..15, addresses its entry), the warps' rings at 128 KB, the partials from
// the start of the dynamic shared memory up to the table (the first
// low_tiles tiles of a chunk) and after the rings (the rest).  The dynamic
// shared memory starts below 1 KB of the window: the host sizes the low
// partials for 63 KB and the high ones for what the rings leave of kDSmem.
static_assert(kDRingAt + DGeom<1>::kRingBytes <= (uint32_t)kDSmem && DGeom<2>::kRingBytes <= DGeom<1>::kRingBytes,
              "shared-memory layout");

template <int kMode, int kNT>
__global__ void __launch_bounds__(kDThreads, 1)
    k_decode(const __nv_bfloat16 *__restrict__ x, int M, int64_t K, int64_t N, const uint8_t *__restrict__ packed,
             const uint8_t *__restrict__ q8, const float *__restrict__ scales, const float *__restrict__ offset,
             const __nv_bfloat16 *__restrict__ Bl, int r, const __nv_bfloat16 *__restrict__ t2, int rp,
             __nv_bfloat16 *__restrict__ y, unsigned *err, int chunk_tiles, int low_tiles) {
    using G = DGeom<kNT>;
    extern __shared__ __align__(16) uint8_t s_dyn[];
    // programmatic dependent launch: see k_gemm_tc.  Without an adapter the
    // kernel waits for the grid before it only after the set-up that reads
    // no global memory (the pair table), and before reading x or W.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int64_t kblocks = K >> 6, row_bytes = K >> 1;
    DWork wk;
    wk.init((uint32_t)((N + 15) >> 4), K, kNT, warp, chunk_tiles, blockIdx.x, gridDim.x);
    const uint32_t s_base = (uint32_t)__cvta_generic_to_shared(s_dyn);
    const uint32_t tile_bytes = (uint32_t)wk.nslot * G::kTileFloats * 4u;
    const uint32_t hi_at = kDRingAt + G::kRingBytes;
    {
        uint32_t dyn_bytes;
        asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(dyn_bytes));
        const uint32_t hi_tiles = chunk_tiles > low_tiles ? (uint32_t)(chunk_tiles - low_tiles) : 0u;
        if (s_base > 1024u || low_tiles < 0 || s_base + (uint32_t)low_tiles * tile_bytes > kDTableAt ||
            s_base + dyn_bytes < hi_at + hi_tiles * tile_bytes) {  // unexpected window: report, touch nothing
            if (threadIdx.x == 0) atomicOr(err, 2u);
            return;
        }
    }
    float *s_part = reinterpret_cast<float *>(s_dyn);
    float *s_hi = reinterpret_cast<float *>(s_dyn + (hi_at - s_base));
    // partial tiles of tile jt of the chunk (nslot slots of kTileFloats)
    auto tile_part = [&](int jt) -> float * {
        return jt < low_tiles ? s_part + jt * wk.nslot * G::kTileFloats
                              : s_hi + (jt - low_tiles) * wk.nslot * G::kTileFloats;
    };

    // this warp's ring; lane l copies 16-byte chunk cc of rows cr + kRowStep i
    constexpr int kLanesPerRow = (int)G::kRowBytes / 16, kRowStep = 32 / kLanesPerRow;
    const uint32_t ring = kDRingAt + (uint32_t)warp * (kDRing * G::kUnitBytes);
    const int cr = lane / kLanesPerRow, cc = lane % kLanesPerRow;
    auto fetch = [&](const DCursor &c, int slot) {
        if (c.valid(wk)) {
            const int64_t row0 = (wk.t0 + c.j) * 16 + cr;
            const int64_t col = (int64_t)c.s * G::kRowBytes + cc * 16;
            const uint32_t dst = ring + (uint32_t)slot * G::kUnitBytes;
#pragma unroll
            for (int i = 0; i < 16 / kRowStep; ++i) {
                const int row = cr + kRowStep * i;
                const bool v = row0 + kRowStep * i < N && col < row_bytes;
                const uint32_t ch = kNT == 1 ? (uint32_t)(cc ^ (row & 7)) : (uint32_t)cc;
                cp_async16(dst + row * G::kRowBytes + (ch << 4),
                           v ? packed + (row0 + kRowStep * i) * row_bytes + col : packed, v);
            }
        }
        cp_async_commit();  // one group per fetch, empty or not: the wait counts stay uniform
    };
    // block constants, loaded two units ahead (raw operands; the three sets
    // rotate by register moves)
    ScaleRaw sr_cur[2], sr_n1[2], sr_n2[2];
    auto load_scales = [&](const DCursor &c, ScaleRaw (&d)[2]) {
        const int64_t bk = (int64_t)G::kBlocksPerUnit * c.s + tq / kNT;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int64_t row = (wk.t0 + c.j) * 16 + g + 8 * i;
            if (c.valid(wk) && row < N && bk < kblocks) {
                d[i] = block_scale_load<kMode>(q8, scales, row * kblocks + bk);
            } else {
                d[i].q8 = 0;
                d[i].v = 0.0f;
            }
        }
    };
    uint2 xr[kNT][G::kXFrags];
    int x_slice = -1;
    auto load_x = [&](int s) {  // x fragments of slice s, tokens g + 8 nt: 128 / kNT contiguous bytes each
        x_slice = s;
        const int64_t col = (int64_t)s * (256 / kNT) + tq * (64 / kNT);
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) {
            const int m = 8 * nt + g;
            const bool xv = m < M && col < K;
            const uint4 *xp = reinterpret_cast<const uint4 *>(x + (xv ? (int64_t)m * K + col : 0));
#pragma unroll
            for (int q = 0; q < G::kXFrags / 2; ++q) {
                const uint4 v = xv ? __ldg(xp + q) : make_uint4(0u, 0u, 0u, 0u);
                xr[nt][2 * q] = make_uint2(v.x, v.y);
                xr[nt][2 * q + 1] = make_uint2(v.z, v.w);
            }
        }
    };
    DCursor c_read, c_fetch, c_sc;
    c_read.start(wk);
    c_fetch = c_read;
    c_sc = c_read;
    // the first copies, block constants and x (reads of global memory)
    auto start_stream = [&]() {
#pragma unroll
        for (int d = 0; d < kDRing; ++d) {
            fetch(c_fetch, d);
            c_fetch.step(wk, warp);
        }
        load_scales(c_sc, sr_cur);
        c_sc.step(wk, warp);
        load_scales(c_sc, sr_n1);
        c_sc.step(wk, warp);
        if (c_read.valid(wk)) load_x(c_read.s);
    };
    {
        // 16 copies of (q[b >> 4], q[b & 15]) in the first 128 bytes of
        // entry b (a 64-bit read by 16 lanes is served at once, so lanes l
        // and l + 16 may share a copy); the levels as immediates (lane i < 16
        // selects level i), spread by shuffles
        static constexpr float kLv[16] = {
            -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
            -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
            0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
            0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};
        float lv = kLv[0];
#pragma unroll
        for (int i = 1; i < 16; ++i) lv = (lane & 15) == i ? kLv[i] : lv;
        // float4 i: entry b = i >> 3, bytes 16 (i & 7) .. of it; b & 15 is
        // the same for all of a thread's float4s
        const float lo = __shfl_sync(0xFFFFFFFFu, lv, (threadIdx.x >> 3) & 15);
        float4 *t4 = reinterpret_cast<float4 *>(s_dyn + (kDTableAt - s_base));
#pragma unroll
        for (int k = 0; k < 256 * 8 / kDThreads; ++k) {
            const int i = threadIdx.x + k * kDThreads, b = i >> 3;
            const float hi = __shfl_sync(0xFFFFFFFFu, lv, b >> 4);
            t4[b * 16 + (i & 7)] = make_float4(hi, lo, hi, lo);
        }
    }
    // with an adapter nothing before this kernel writes what it reads (the
    // down-projection before it releases it only after its own wait), so
    // only its epilogue waits; without one x and W wait for the grid before
    if (r <= 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    __syncthreads();  // the pair table is complete
    // each warp starts its stream after the barrier, so that no warp waits
    // for the others to have issued their first copies (the copy queue is
    // full for ~1.4 us as every SM asks for 3 units per warp at once)
    start_stream();

    const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
    const uint32_t base_lane = kDTableAt | (uint32_t)((lane & 15) * 8);
    // lane's two rows in a unit: g and g + 8 (same swizzle phase); kNT = 1:
    // chunks 2 tq, 2 tq + 1 of 128-byte rows, kNT = 2: chunk tq of 64-byte rows
    const uint32_t off0 = kNT == 1 ? (uint32_t)g * 128u + ((uint32_t)((2 * tq) ^ g) << 4)
                                   : (uint32_t)g * 64u + ((uint32_t)tq << 4);
    const uint32_t off1 = (uint32_t)g * 128u + ((uint32_t)((2 * tq + 1) ^ g) << 4);

    int u = 0;  // units consumed by this warp
    for (int c0 = 0; c0 < wk.my_tiles; c0 += chunk_tiles) {
        const int c1 = wk.my_tiles - c0 < chunk_tiles ? wk.my_tiles : c0 + chunk_tiles;
        for (; c_read.valid(wk) && c_read.j < c1; ++u) {
            load_scales(c_sc, sr_n2);
            c_sc.step(wk, warp);
            const int j = c_read.j, s = c_read.s;
            if (s != x_slice) load_x(s);
            // unit u's copies (this thread's) are complete once at most
            // kDRing - 1 later groups pend; the warp's after the barrier
            asm volatile("cp.async.wait_group %0;" ::"n"(kDRing - 1) : "memory");
            __syncwarp();
            const int slot = u % kDRing;
            const uint32_t ub = ring + (uint32_t)slot * G::kUnitBytes;
            uint32_t w[2][G::kWords];
            {
                constexpr uint32_t kHalf = 8 * G::kRowBytes;  // row g + 8
                uint4 a0, b0;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a0.x), "=r"(a0.y), "=r"(a0.z), "=r"(a0.w) : "r"(ub + off0));
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(b0.x), "=r"(b0.y), "=r"(b0.z), "=r"(b0.w) : "r"(ub + kHalf + off0));
                w[0][0] = a0.x, w[0][1] = a0.y, w[0][2] = a0.z, w[0][3] = a0.w;
                w[1][0] = b0.x, w[1][1] = b0.y, w[1][2] = b0.z, w[1][3] = b0.w;
                if constexpr (kNT == 1) {
                    uint4 a1, b1;
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(a1.x), "=r"(a1.y), "=r"(a1.z), "=r"(a1.w) : "r"(ub + off1));
                    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(b1.x), "=r"(b1.y), "=r"(b1.z), "=r"(b1.w) : "r"(ub + kHalf + off1));
                    w[0][4] = a1.x, w[0][5] = a1.y, w[0][6] = a1.z, w[0][7] = a1.w;
                    w[1][4] = b1.x, w[1][5] = b1.y, w[1][6] = b1.z, w[1][7] = b1.w;
                }
            }
            __syncwarp();  // every lane has read the slot: refill it
            fetch(c_fetch, slot);
            c_fetch.step(wk, warp);

            const float sc0 = block_scale_finish<kMode>(sr_cur[0], mu);
            const float sc1 = block_scale_finish<kMode>(sr_cur[1], mu);
            float acc[kNT][G::kChains][4];
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                for (int ch = 0; ch < G::kChains; ++ch)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[nt][ch][i] = 0.0f;
            mma_unit<kNT>(w, sc0, sc1, base_lane, xr, acc);
            const int sl = c_read.slot(wk, warp);
            float *pp = tile_part(j - c0) + sl * G::kTileFloats + lane;
            if (s < kDWarps) {
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        pp[128 * nt + 32 * i] = G::kChains == 1 ? acc[nt][0][i] : acc[nt][0][i] + acc[nt][G::kChains - 1][i];
            } else {
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        pp[128 * nt + 32 * i] += G::kChains == 1 ? acc[nt][0][i] : acc[nt][0][i] + acc[nt][G::kChains - 1][i];
            }
            c_read.step(wk, warp);
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                sr_cur[i] = sr_n1[i];
                sr_n1[i] = sr_n2[i];
            }
        }
        __syncthreads();
        const int nt_chunk = c1 - c0;
        // add the slots of every tile in slot order (in place, into slot 0)
        for (int e = threadIdx.x; e < nt_chunk * G::kTileFloats; e += kDThreads) {
            const int jt = e / G::kTileFloats, el = e % G::kTileFloats;
            float *p = tile_part(jt) + el;
            float v = p[0];
            for (int sl = 1; sl < wk.nslot; ++sl) v += p[sl * G::kTileFloats];
            if (r > 0) {
                p[0] = v;
            } else {
                const int i = (el >> 5) & 3, ln = el & 31;
                const int64_t n = (wk.t0 + c0 + jt) * 16 + (ln >> 2) + 8 * (i >> 1);
                const int m = 8 * (el >> 7) + 2 * (ln & 3) + (i & 1);
                if (n < N && m < M) y[(int64_t)m * N + n] = __float2bfloat16_rn(v);
            }
        }
        if (r > 0) {
            __syncthreads();
            // t is written by the down-projection kernel launched just before
            // this one (programmatic dependent launch): wait for it only here.
            asm volatile("griddepcontrol.wait;" ::: "memory");
            for (int jt = warp; jt < nt_chunk; jt += kDWarps) {
                const float *p = tile_part(jt) + lane;
                float acc[kNT][4];
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[nt][i] = p[128 * nt + 32 * i];
                const int64_t row0 = (wk.t0 + c0 + jt) * 16 + g, row1 = row0 + 8;
                const bool rv0 = row0 < N, rv1 = row1 < N;
                const uint32_t *ba = reinterpret_cast<const uint32_t *>(Bl + (rv0 ? row0 : 0) * r);
                const uint32_t *bb = reinterpret_cast<const uint32_t *>(Bl + (rv1 ? row1 : 0) * r);
                for (int js = 0; js < (2 * r) / 16; ++js) {
                    const int w0 = (((16 * js) % r) + 2 * tq) >> 1;
                    uint32_t a[4];
                    a[0] = rv0 ? __ldg(ba + w0) : 0u;
                    a[1] = rv1 ? __ldg(bb + w0) : 0u;
                    a[2] = rv0 ? __ldg(ba + w0 + 4) : 0u;
                    a[3] = rv1 ? __ldg(bb + w0 + 4) : 0u;
                    const int tw = (16 * js + 2 * tq) >> 1;
#pragma unroll
                    for (int nt = 0; nt < kNT; ++nt) {
                        const int m = 8 * nt + g;
                        const bool tv = m < M;
                        const uint32_t *tr = reinterpret_cast<const uint32_t *>(t2 + (int64_t)(tv ? m : 0) * rp);
                        // L2-coherent loads: t was written by the preceding kernel
                        const uint32_t tb0 = tv ? __ldcg(tr + tw) : 0u, tb1 = tv ? __ldcg(tr + tw + 4) : 0u;
                        mma_bf16_16816(acc[nt], a, tb0, tb1);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int64_t n = (i >> 1) ? row1 : row0;
                        const int m = 8 * nt + 2 * tq + (i & 1);
                        if (n < N && m < M) y[(int64_t)m * N + n] = __float2bfloat16_rn(acc[nt][i]);
                    }
            }
        }
        __syncthreads();  // partials are rewritten next
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // no copy outlives the CTA
}

template <int kMode, int kNT>
cudaError_t launch_decode_mode(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                               const float *scales, const float *offset, const void *B, int r, const void *t2,
                               int rp, void *y, unsigned *err, cudaStream_t stream, int grid, int chunk,
                               int low_tiles) {
    cudaError_t e = cudaFuncSetAttribute(k_decode<kMode, kNT>, cudaFuncAttributeMaxDynamicSharedMemorySize, kDSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_decode<kMode, kNT>, dim3(grid), dim3(kDThreads), (size_t)kDSmem, stream, 1,
                      static_cast<const __nv_bfloat16 *>(x), M, K, N, packed, q8, scales, offset,
                      static_cast<const __nv_bfloat16 *>(B), r, static_cast<const __nv_bfloat16 *>(t2), rp,
                      static_cast<__nv_bfloat16 *>(y), err, chunk, low_tiles);
}

template <int kNT>
cudaError_t launch_decode_nt(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                             const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                             void *y, unsigned *err, cudaStream_t stream, int num_sms) {
    DChunk ch;
    if (!decode_chunk(N, K, kNT, num_sms, &ch)) return cudaErrorInvalidValue;
    if (q8 == nullptr)
        return launch_decode_mode<2, kNT>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, err, stream,
                                          ch.grid, ch.chunk, ch.low_tiles);
    if (offset == nullptr)
        return launch_decode_mode<1, kNT>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, err, stream,
                                          ch.grid, ch.chunk, ch.low_tiles);
    return launch_decode_mode<0, kNT>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, err, stream, ch.grid,
                                      ch.chunk, ch.low_tiles);
}

}  // namespace

// Decode kernel for 1 <= M <= 16 (K a multiple of 64, pointers 16-byte
// aligned): one token tile of 8 up to M = 8, two above; num_sms: SMs the
// grid may take.
cudaError_t launch_decode(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                          const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                          void *y, unsigned *err, cudaStream_t stream, int num_sms) {
    if (M < 1 || M > 16 || K < 64 || (K & 63) != 0 || N < 1 || num_sms < 1) return cudaErrorInvalidValue;
    if (M <= 8)
        return launch_decode_nt<1>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, err, stream, num_sms);
    return launch_decode_nt<2>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, err, stream, num_sms);
}

}  // namespace nf4
