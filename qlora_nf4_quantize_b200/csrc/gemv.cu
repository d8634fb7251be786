// gemv.cu -- K4: fused NF4-dequantizing linear for small token counts
// (M <= 16; the dispatcher, linear.cu, sends 9 to 16 tokens to the
// tensor-core pipeline's 16-token tile instead), y = x W~^T + [t_hi | t_lo]
// [B | B]^T.
//
// "QLoRA: Mathematical Foundations ...", section "Forward Pass Computation":
// the weight is dequantized on the fly into registers and never written to
// memory; compute dtype bf16 with fp32 accumulation.  The W~ values are
// exactly the bf16 outputs of nf4_dequantize (RNE_bf16(RN_f32(q * c1'))).
//
// The kernel streams the packed weight once from HBM (0.5 B + 1/64 B per
// parameter) and is designed to be bound by that stream.
//
// Work layout
//   - A CTA (4 warps) owns a tile of 16 (T <= 8) or 32 (T > 8) weight rows;
//     the warps split K in
//     super-steps of 256 columns (warp w takes super-steps w, w+4, ...) and
//     their partial sums are added in shared memory in warp order.  Each
//     warp keeps the next super-step's codes and scales in flight while it
//     computes the current one.
//   - Each warp runs m16n8k16 tensor-core MMAs with the weight as the A
//     operand (one m16 tile per 16 rows) and x as the B operand (one n8 tile
//     per 8 tokens; x is read through L1).  Within a super-step the K index is permuted so that the four
//     A-fragment columns a lane owns at MMA step s (2t, 2t+1, 2t+8, 2t+9) are
//     elements 4s..4s+3 of 64-block t of its rows; the x fragment uses the
//     same permutation (one 8-byte load of x[token, 64 t + 4 s ...]).  So a
//     lane dequantizes whole 64-blocks: one scale and one register lookup
//     table (mma_util.cuh, make_lut) per block, then 3 byte permutes per
//     weight and no shared memory.
//   - The LoRA term is a K-extension of 2r columns after the reduction, and
//     the CTA writes its 16 x M outputs.
#include "mma_util.cuh"

namespace nf4 {
namespace {

#ifndef NF4_GEMV_WARPS
#define NF4_GEMV_WARPS 4
#endif
constexpr int kGemvWarps = NF4_GEMV_WARPS;
// Resident CTAs per SM the register allocation of the one-token-tile
// kernel must allow: 5 caps it at 102 registers (it needs 95, no spills), so
// the 688 tiles of an 11008-row weight run as one wave of 740 slots instead
// of 1.5 waves of 444 (148 registers): 17.0 -> 16.5 us without LoRA, 18.9
// -> 18.0 us with r = 16 at one token.  The two-token-tile instantiation
// spills under that cap and keeps the default.
#ifndef NF4_GEMV_MINB
#define NF4_GEMV_MINB 5
#endif
// 0 = register lookup table, 1 = shared-memory pair table, 2 = pair table for
// the first row of each m16 tile and register table for the second
#ifndef NF4_GEMV_SMEM_LUT
#define NF4_GEMV_SMEM_LUT 0
#endif
constexpr int kGemvLut = NF4_GEMV_SMEM_LUT;
constexpr bool kGemvSmemLut = NF4_GEMV_SMEM_LUT != 0;

// Packed codes (8 words = one 64-block) and block constants of the 2 MT rows a
// lane owns in one super-step; all-zero-code words outside the matrix.
template <int MT>
struct BlockSet {
    uint32_t w[2 * MT][8];
    ScaleRaw sr[2 * MT];  // block constant operands (decoded at use)
};

template <int kMode, int MT>
__device__ __forceinline__ void load_set(const uint8_t *__restrict__ packed, const uint8_t *__restrict__ q8,
                                         const float *__restrict__ scales, float /*mu*/, const int64_t *row,
                                         const bool *rvalid, int64_t K, int64_t kblocks, int64_t bk,
                                         BlockSet<MT> &bp) {
    const bool kvalid = bk < kblocks;
#pragma unroll
    for (int i = 0; i < 2 * MT; ++i) {
        if (rvalid[i] && kvalid) {
            const uint4 *p = reinterpret_cast<const uint4 *>(packed + row[i] * (K >> 1) + bk * 32);
            const uint4 u0 = __ldg(p), u1 = __ldg(p + 1);
            bp.w[i][0] = u0.x; bp.w[i][1] = u0.y; bp.w[i][2] = u0.z; bp.w[i][3] = u0.w;
            bp.w[i][4] = u1.x; bp.w[i][5] = u1.y; bp.w[i][6] = u1.z; bp.w[i][7] = u1.w;
            bp.sr[i] = block_scale_load<kMode>(q8, scales, row[i] * kblocks + bk);
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) bp.w[i][j] = 0x77777777u;
            bp.sr[i].q8 = 0;
            bp.sr[i].v = 0.0f;
        }
    }
}

// kSmemLut: dequantize through the shared-memory pair table (mma_util.cuh,
// pair_lookup4: one byte permute, one shared load and two multiplies per two
// weights) instead of the per-block register lookup table (lut_lookup4: about
// three byte permutes per weight, all on the integer pipe).
template <int kMode, int NT, int MT, int kLutSel>
__global__ void __launch_bounds__(kGemvWarps * 32, MT == 1 ? NF4_GEMV_MINB : 1) k_gemv(const __nv_bfloat16 *__restrict__ x, int M, int64_t K,
                                                          int64_t N, const uint8_t *__restrict__ packed,
                                                          const uint8_t *__restrict__ q8,
                                                          const float *__restrict__ scales,
                                                          const float *__restrict__ offset,
                                                          const __nv_bfloat16 *__restrict__ Bl, int r,
                                                          const __nv_bfloat16 *__restrict__ t2, int rp,
                                                          __nv_bfloat16 *__restrict__ y) {
    constexpr bool kSmemLut = kLutSel != 0;
    // programmatic dependent launch: see k_gemm_tc (x and W at once when the
    // down-projection precedes; otherwise wait before reading anything)
    if (r <= 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ float s_part[kGemvWarps][MT][NT][4][32];
    extern __shared__ float2 s_pairs[];  // kPairTableFloat2 entries when kSmemLut
    if constexpr (kSmemLut) {
        fill_pair_table(s_pairs);
        __syncthreads();
    }
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float2 *tbl_lane = s_pairs + (lane & 15);
    const int g = lane >> 2, tq = lane & 3;
    const int64_t n0 = (int64_t)blockIdx.x * (16 * MT);
    const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
    const int64_t kblocks = K >> 6;             // 64-blocks per row
    const int64_t nsuper = (kblocks + 3) >> 2;  // super-steps of 4 blocks

    // rows owned by this lane: n0 + g + 8 i; m16 tile mt holds rows 2 mt, 2 mt + 1
    int64_t row[2 * MT];
    bool rvalid[2 * MT];
#pragma unroll
    for (int i = 0; i < 2 * MT; ++i) {
        row[i] = n0 + g + 8 * i;
        rvalid[i] = row[i] < N;
    }
    // token rows of the x fragments: token g + 8 nt
    const uint2 *xrow[NT];
    bool tvalid[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int tok = g + 8 * nt;
        tvalid[nt] = tok < M;
        xrow[nt] = reinterpret_cast<const uint2 *>(x + (int64_t)(tvalid[nt] ? tok : 0) * K);
    }

    float acc[MT][NT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.0f;

    // software pipeline: the next super-step's codes and scales are in flight
    // while the current one is dequantized and multiplied
    BlockSet<MT> cur, nxt;
    int64_t ss = warp;
    if (ss < nsuper) load_set<kMode, MT>(packed, q8, scales, mu, row, rvalid, K, kblocks, ss * 4 + tq, cur);
    for (; ss < nsuper; ss += kGemvWarps) {
        const int64_t bk = ss * 4 + tq;  // this lane's 64-block along K
        const bool kvalid = bk < kblocks;
        if (ss + kGemvWarps < nsuper)
            load_set<kMode, MT>(packed, q8, scales, mu, row, rvalid, K, kblocks, (ss + kGemvWarps) * 4 + tq, nxt);
        float cs[2 * MT];
#pragma unroll
        for (int i = 0; i < 2 * MT; ++i) cs[i] = block_scale_finish<kMode>(cur.sr[i], mu);
        Lut lut[2 * MT];
        if constexpr (kLutSel != 1) {
#pragma unroll
            for (int i = (kLutSel == 2 ? 1 : 0); i < 2 * MT; i += (kLutSel == 2 ? 2 : 1)) lut[i] = make_lut(cs[i]);
        }
        const int64_t kx4 = bk * 16;  // x offset of this block in 4-element units
#pragma unroll
        for (int s = 0; s < 16; ++s) {
            uint2 xb[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) xb[nt] = (tvalid[nt] && kvalid) ? __ldg(xrow[nt] + kx4 + s) : make_uint2(0u, 0u);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                const uint32_t p0 = cur.w[2 * mt][s >> 1] >> ((s & 1) * 16);
                const uint32_t p1 = cur.w[2 * mt + 1][s >> 1] >> ((s & 1) * 16);
                if constexpr (kLutSel == 1) {
                    pair_lookup4(tbl_lane, p0, cs[2 * mt], a[0], a[2]);
                    pair_lookup4(tbl_lane, p1, cs[2 * mt + 1], a[1], a[3]);
                } else if constexpr (kLutSel == 2) {
                    pair_lookup4(tbl_lane, p0, cs[2 * mt], a[0], a[2]);
                    lut_lookup4(lut[2 * mt + 1], p1, a[1], a[3]);
                } else {
                    lut_lookup4(lut[2 * mt], p0, a[0], a[2]);
                    lut_lookup4(lut[2 * mt + 1], p1, a[1], a[3]);
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[mt][nt], a, xb[nt].x, xb[nt].y);
            }
        }
        cur = nxt;
    }

#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) s_part[warp][mt][nt][i][lane] = acc[mt][nt][i];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v = s_part[0][mt][nt][i][lane];
#pragma unroll
                for (int w = 1; w < kGemvWarps; ++w) v += s_part[w][mt][nt][i][lane];
                acc[mt][nt][i] = v;
            }

    // LoRA K-extension: 2r columns, A operand = [B | B] rows, B operand = [t_hi | t_lo]
    if (r > 0) {
        // t is written by the down-projection kernel launched just before this
        // one (programmatic dependent launch): wait for it only here.
        asm volatile("griddepcontrol.wait;" ::: "memory");
        for (int js = 0; js < (2 * r) / 16; ++js) {
            const int j0 = (16 * js) % r;  // column of B for k-slot 0 of this step
            uint32_t tb0[NT], tb1[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const uint32_t *tr = reinterpret_cast<const uint32_t *>(t2 + (int64_t)(g + 8 * nt) * rp);
                const int w0 = (16 * js + 2 * tq) >> 1;
                // L2-coherent loads: t was written by the preceding kernel
                tb0[nt] = tvalid[nt] ? __ldcg(tr + w0) : 0u;
                tb1[nt] = tvalid[nt] ? __ldcg(tr + w0 + 4) : 0u;
            }
            const int w0 = (j0 + 2 * tq) >> 1;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const uint32_t *ba = reinterpret_cast<const uint32_t *>(Bl + (rvalid[2 * mt] ? row[2 * mt] : 0) * r);
                const uint32_t *bb =
                    reinterpret_cast<const uint32_t *>(Bl + (rvalid[2 * mt + 1] ? row[2 * mt + 1] : 0) * r);
                uint32_t a[4];
                a[0] = rvalid[2 * mt] ? __ldg(ba + w0) : 0u;
                a[1] = rvalid[2 * mt + 1] ? __ldg(bb + w0) : 0u;
                a[2] = rvalid[2 * mt] ? __ldg(ba + w0 + 4) : 0u;
                a[3] = rvalid[2 * mt + 1] ? __ldg(bb + w0 + 4) : 0u;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[mt][nt], a, tb0[nt], tb1[nt]);
            }
        }
    }

    // D fragment: d0, d1 = (row g, tokens 2tq, 2tq+1), d2, d3 = (row g + 8, ...)
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t n = row[2 * mt + (i >> 1)];
                const int m = 8 * nt + 2 * tq + (i & 1);
                if (n < N && m < M) y[(int64_t)m * N + n] = __float2bfloat16_rn(acc[mt][nt][i]);
            }
}

// ---------------------------------------------------------------------------
// Persistent variant (K % 256 == 0 and x fits in shared memory): one CTA of
// 16 warps per SM walks 16-row weight tiles (tile = blockIdx.x + i gridDim.x).
//   - Work unit = (tile, super-step ss): 256 columns of packed codes (16 rows
//     x 128 bytes) plus the block constants' raw operands.  Warp w takes the
//     units of tile i with (ss + i) % 16 == w.
//   - Each warp streams its units through its own ring of D slots in shared
//     memory with cp.async, D units ahead of the one it computes (D from the
//     shared memory left over, 2..8); 16-byte chunks are XOR-swizzled by row
//     so that the fragment reads are conflict-free.
//   - x (M rows, compact, in MMA-fragment order: one conflict-free 128-bit
//     load per fragment pair) is staged once per CTA.
//   - Per tile the 16 warps' partial tiles meet in shared memory and every
//     thread adds one output's 16 partials in warp order.  Without LoRA the
//     sum is stored; with LoRA it is kept (fp32, shared memory) and, once all
//     tiles are done, the down-projection's t is awaited and staged and each
//     tile's K-extension of 2r columns is added by MMA before the store, so
//     the down-projection runs entirely under the main loop.
//   - kLut: 0 = register lookup table (integer pipe), 1 = shared-memory pair
//     table (shared-memory pipe), 2 = pair table for a lane's first row and
//     register table for its second, spreading the work over both pipes.
constexpr int kPWarps = 16;
constexpr int kPSlotBytes = 2048 + 256;  // codes + block constants

__host__ __device__ constexpr int gemv_p_t2_stride(int rp) { return rp + 8; }  // bf16 per staged t row

struct GemvPLayout {
    int64_t x_off, t2_off, res_off, part_off, pair_off, ring_off, total;
};

// my_tiles_max: most tiles one CTA walks (kept results, LoRA only)
__host__ __device__ inline GemvPLayout gemv_p_layout(int M, int64_t K, int rp, int nt, bool smem_lut, int depth,
                                                     int my_tiles_max) {
    GemvPLayout L;
    L.x_off = 0;
    L.t2_off = L.x_off + (int64_t)M * K * 2;
    L.res_off = L.t2_off + (rp > 0 ? (int64_t)M * gemv_p_t2_stride(rp) * 2 : 0);
    L.res_off = (L.res_off + 15) & ~(int64_t)15;
    L.part_off = L.res_off + (rp > 0 ? (int64_t)my_tiles_max * nt * 128 * 4 : 0);
    L.pair_off = L.part_off + (int64_t)kPWarps * nt * 4 * 32 * 4;
    L.ring_off = L.pair_off + (smem_lut ? kPairTableFloat2 * (int64_t)sizeof(float2) : 0);
    L.total = L.ring_off + (int64_t)kPWarps * depth * kPSlotBytes;
    return L;
}

// cp.async of `bytes` (4 or 16) with zero fill when !valid
template <int kBytes>
__device__ __forceinline__ void cp_async(void *dst, const void *src, bool valid) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    if constexpr (kBytes == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(valid ? 16 : 0) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(d), "l"(src), "r"(valid ? 4 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most n (0..8) of this thread's groups are pending
__device__ __forceinline__ void cp_async_wait_dyn(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
        case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
        case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
        case 7: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 8;" ::: "memory"); break;
    }
}

// The sequence of units of one warp: tiles in order, within a tile the
// super-steps ss = (w - i) mod 16, + 16, ... below nsuper.
struct UnitIter {
    int tile_i, ss;
    __device__ __forceinline__ void settle(int w, int my_tiles, int nsuper) {
        while (tile_i < my_tiles && ss >= nsuper) {
            ++tile_i;
            ss = ((w - tile_i) % kPWarps + kPWarps) % kPWarps;
        }
    }
    __device__ __forceinline__ void start(int w, int my_tiles, int nsuper) {
        tile_i = 0;
        ss = w;
        settle(w, my_tiles, nsuper);
    }
    __device__ __forceinline__ void next(int w, int my_tiles, int nsuper) {
        ss += kPWarps;
        settle(w, my_tiles, nsuper);
    }
};

template <int kMode, int NT, int kLut>
__global__ void __launch_bounds__(kPWarps * 32, 1)
    k_gemv_p(const __nv_bfloat16 *__restrict__ x, int M, int64_t K, int64_t N, const uint8_t *__restrict__ packed,
             const uint8_t *__restrict__ q8, const float *__restrict__ scales, const float *__restrict__ offset,
             const __nv_bfloat16 *__restrict__ Bl, int r, const __nv_bfloat16 *__restrict__ t2, int rp,
             __nv_bfloat16 *__restrict__ y, int depth, int my_tiles_max) {
    extern __shared__ __align__(16) uint8_t s_dyn[];
    // programmatic dependent launch: see k_gemm_tc
    if (r <= 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr bool kSmemLut = kLut != 0;
    const GemvPLayout L = gemv_p_layout(M, K, rp, NT, kSmemLut, depth, my_tiles_max);
    uint4 *xs = reinterpret_cast<uint4 *>(s_dyn + L.x_off);
    __nv_bfloat16 *t2s = reinterpret_cast<__nv_bfloat16 *>(s_dyn + L.t2_off);
    float *s_res = reinterpret_cast<float *>(s_dyn + L.res_off);
    float *s_part = reinterpret_cast<float *>(s_dyn + L.part_off);
    const float2 *s_pairs = reinterpret_cast<const float2 *>(s_dyn + L.pair_off);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    uint8_t *ring = s_dyn + L.ring_off + (int64_t)warp * depth * kPSlotBytes;
    const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
    const int64_t kblocks = K >> 6;
    const int nsuper = (int)(kblocks >> 2);
    const int64_t n_tiles = (N + 15) >> 4;
    const int my_tiles = (int)((n_tiles - 1 - blockIdx.x) / gridDim.x + 1);

    // Copies of one unit, per lane: code chunk `ch` of rows ch_row + 4 i
    // (i = 0..3, 8 lanes per 128-byte row) and the block constants of row
    // lane & 15.  The row pointers change only with the tile.
    const int ch = lane & 7, ch_row = lane >> 3, sc_row = lane & 15;
    int staged_tile = -1;
    const uint8_t *code_src[4];
    bool code_ok[4];
    const uint8_t *sc_src = nullptr;
    int64_t sc_b = 0;  // first block of row lane & 15
    bool sc_ok = false;
    auto stage = [&](const UnitIter &it, int slot) {
        if (it.tile_i < my_tiles) {
            if (it.tile_i != staged_tile) {
                staged_tile = it.tile_i;
                const int64_t row0 = ((int64_t)blockIdx.x + (int64_t)it.tile_i * gridDim.x) * 16;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int64_t n = row0 + ch_row + 4 * i;
                    code_ok[i] = n < N;
                    code_src[i] = packed + (code_ok[i] ? n : 0) * (K >> 1) + ch * 16;
                }
                const int64_t n = row0 + sc_row;
                sc_ok = n < N;
                sc_b = (sc_ok ? n : 0) * kblocks;
                if constexpr (kMode == 2) sc_src = reinterpret_cast<const uint8_t *>(scales + sc_b);
                else sc_src = q8 + sc_b;
            }
            uint8_t *sb = ring + slot * kPSlotBytes;
            const int64_t kb = (int64_t)it.ss * 128;  // byte offset of the unit in a packed row
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int row = ch_row + 4 * i;
                cp_async<16>(sb + (row * 8 + (ch ^ (row & 7))) * 16, code_src[i] + kb, code_ok[i]);
            }
            if constexpr (kMode == 2) {  // fp32 constants: 16 bytes per row
                if (lane < 16) cp_async<16>(sb + 2048 + lane * 16, sc_src + it.ss * 16, sc_ok);
            } else {  // E4M3 codes (4 bytes per row) and the row's c2 (the same for the unit's 4 blocks)
                if (lane < 16) cp_async<4>(sb + 2048 + sc_row * 4, sc_src + it.ss * 4, sc_ok);
                else cp_async<4>(sb + 2048 + 64 + sc_row * 4, scales + ((sc_b + it.ss * 4) >> 8), sc_ok);
            }
        }
        cp_async_commit();
    };

    // prologue: x (one group), then the first `depth` units
    {
        const int64_t kchunks = K >> 3;
        const int64_t total = (int64_t)M * kchunks;
        for (int64_t c = threadIdx.x; c < total; c += blockDim.x) {
            const int tok = (int)(c / kchunks);
            const int64_t k = (c - (int64_t)tok * kchunks) * 8;
            const int64_t ss = k >> 8;
            const int t = (int)((k >> 6) & 3), p = (int)((k >> 3) & 7);
            cp_async<16>(xs + ((ss * 8 + p) * M + tok) * 4 + t, x + (int64_t)tok * K + k, true);
        }
        cp_async_commit();
    }
    UnitIter issue, cons;
    issue.start(warp, my_tiles, nsuper);
    cons = issue;
    for (int d = 0; d < depth; ++d) {
        stage(issue, d);
        issue.next(warp, my_tiles, nsuper);
    }
    if constexpr (kSmemLut) fill_pair_table(const_cast<float2 *>(s_pairs));
    const uint32_t tbl_lane = (uint32_t)__cvta_generic_to_shared(s_pairs + (lane & 15));
    cp_async_wait_dyn(depth);  // x complete (the `depth` unit groups may pend)
    __syncthreads();           // x and the table visible to all

    int u = 0;  // units consumed by this warp
    for (int tile_i = 0; tile_i < my_tiles; ++tile_i) {
        float accs[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) accs[nt][0] = accs[nt][1] = accs[nt][2] = accs[nt][3] = 0.0f;
        while (cons.tile_i == tile_i) {
            cp_async_wait_dyn(depth - 1);  // pending: units u+1 .. u+depth-1
            __syncwarp();
            const int slot = u % depth;
            const uint8_t *sb = ring + slot * kPSlotBytes;
            const uint4 *wb = reinterpret_cast<const uint4 *>(sb);
            uint32_t w[2][8];
            ScaleRaw sr[2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int row = g + 8 * i;
                const uint4 c0 = wb[row * 8 + ((2 * tq) ^ (row & 7))];
                const uint4 c1 = wb[row * 8 + ((2 * tq + 1) ^ (row & 7))];
                w[i][0] = c0.x; w[i][1] = c0.y; w[i][2] = c0.z; w[i][3] = c0.w;
                w[i][4] = c1.x; w[i][5] = c1.y; w[i][6] = c1.z; w[i][7] = c1.w;
                if constexpr (kMode == 2) {
                    sr[i].q8 = 0;
                    sr[i].v = reinterpret_cast<const float *>(sb + 2048)[row * 4 + tq];
                } else {
                    sr[i].q8 = sb[2048 + row * 4 + tq];
                    sr[i].v = reinterpret_cast<const float *>(sb + 2048 + 64)[row];
                }
            }
            __syncwarp();  // slot free: refill it with the unit `depth` ahead
            stage(issue, slot);
            issue.next(warp, my_tiles, nsuper);

            const float c0 = block_scale_finish<kMode>(sr[0], mu);
            const float c1 = block_scale_finish<kMode>(sr[1], mu);
            const uint64_t cc0 = pack_f32x2(c0, c0), cc1 = pack_f32x2(c1, c1);
            Lut lut0, lut1;
            if constexpr (kLut == 0) lut0 = make_lut(c0);
            if constexpr (kLut != 1) lut1 = make_lut(c1);
            const uint4 *xq = xs + ((int64_t)cons.ss * 8 * M) * 4 + tq;
#pragma unroll
            for (int q = 0; q < 8; ++q) {  // packed word q = MMA steps 2q, 2q+1
                uint32_t wa[4], wbb[4];
                if constexpr (kLut == 0) {
                    lut_lookup8(lut0, w[0][q], wa);
                } else {
                    pair_lookup4_s(tbl_lane, w[0][q], cc0, wa[0], wa[1]);
                    pair_lookup4_s(tbl_lane, w[0][q] >> 16, cc0, wa[2], wa[3]);
                }
                if constexpr (kLut == 1) {
                    pair_lookup4_s(tbl_lane, w[1][q], cc1, wbb[0], wbb[1]);
                    pair_lookup4_s(tbl_lane, w[1][q] >> 16, cc1, wbb[2], wbb[3]);
                } else {
                    lut_lookup8(lut1, w[1][q], wbb);
                }
                uint4 xv[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int tok = g + 8 * nt;
                    xv[nt] = tok < M ? xq[(q * M + tok) * 4] : make_uint4(0u, 0u, 0u, 0u);
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t a[4] = {wa[2 * h], wbb[2 * h], wa[2 * h + 1], wbb[2 * h + 1]};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        const uint32_t b0 = h ? xv[nt].z : xv[nt].x, b1 = h ? xv[nt].w : xv[nt].y;
                        mma_bf16_16816(accs[nt], a, b0, b1);
                    }
                }
            }
            ++u;
            cons.next(warp, my_tiles, nsuper);
        }
        // the 16 partial tiles meet in shared memory; thread e adds output e's
        // partials in warp order
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) s_part[((warp * NT + nt) * 4 + i) * 32 + lane] = accs[nt][i];
        __syncthreads();
        if (threadIdx.x < NT * 128) {
            const int e = threadIdx.x;
            float v = 0.0f;
#pragma unroll
            for (int ww = 0; ww < kPWarps; ++ww) v += s_part[ww * NT * 128 + e];
            if (r > 0) {
                s_res[tile_i * NT * 128 + e] = v;
            } else {
                const int nt = e >> 7, i = (e >> 5) & 3, ln = e & 31;
                const int64_t n = ((int64_t)blockIdx.x + (int64_t)tile_i * gridDim.x) * 16 + (ln >> 2) + 8 * (i >> 1);
                const int m = 8 * nt + 2 * (ln & 3) + (i & 1);
                if (n < N && m < M) y[(int64_t)m * N + n] = __float2bfloat16_rn(v);
            }
        }
        __syncthreads();  // s_part is rewritten by the next tile
    }
    cp_async_wait_dyn(0);
    if (r <= 0) return;

    // LoRA K-extension of every tile: 2r columns, A = [B | B] (column j ->
    // B[:, j % r]), B operand = [t_hi | t_lo], accumulated onto the kept sums.
    // t is written by the down-projection kernel launched just before this
    // one (programmatic dependent launch): wait for it only here.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int t2_stride = gemv_p_t2_stride(rp);
    {
        const int cpr = (2 * r + 7) >> 3;  // 16-byte chunks of a row of t actually read
        for (int c = threadIdx.x; c < M * cpr; c += blockDim.x) {
            const int tok = c / cpr, ch = c - tok * cpr;
            cp_async<16>(t2s + tok * t2_stride + ch * 8, t2 + (int64_t)tok * rp + ch * 8, true);
        }
        cp_async_commit();
        cp_async_wait_dyn(0);
        __syncthreads();
    }
    for (int tile_i = warp; tile_i < my_tiles; tile_i += kPWarps) {
        const int64_t tile = (int64_t)blockIdx.x + (int64_t)tile_i * gridDim.x;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[nt][i] = s_res[tile_i * NT * 128 + (nt * 4 + i) * 32 + lane];
        const int64_t row0 = tile * 16 + g, row1 = row0 + 8;
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
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int tok = g + 8 * nt;
                const uint32_t *tr = reinterpret_cast<const uint32_t *>(t2s + tok * t2_stride);
                const int tw = (16 * js + 2 * tq) >> 1;
                const uint32_t tb0 = tok < M ? tr[tw] : 0u, tb1 = tok < M ? tr[tw + 4] : 0u;
                mma_bf16_16816(acc[nt], a, tb0, tb1);
            }
        }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t n = (i >> 1) ? row1 : row0;
                const int m = 8 * nt + 2 * tq + (i & 1);
                if (n < N && m < M) y[(int64_t)m * N + n] = __float2bfloat16_rn(acc[nt][i]);
            }
    }
}

template <int kMode, int NT, int kLut>
cudaError_t launch_gemv_p(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                          const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                          void *y, cudaStream_t stream, int num_sms, int depth, size_t smem) {
    cudaError_t e = cudaFuncSetAttribute(k_gemv_p<kMode, NT, kLut>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (N + 15) / 16;
    const int64_t grid = tiles < num_sms ? tiles : num_sms;  // num_sms: SMs this grid may take
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kPWarps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_gemv_p<kMode, NT, kLut>, static_cast<const __nv_bfloat16 *>(x), M, K, N,
                              packed, q8, scales, offset, static_cast<const __nv_bfloat16 *>(B), r,
                              static_cast<const __nv_bfloat16 *>(t2), rp, static_cast<__nv_bfloat16 *>(y), depth,
                              (int)((tiles + grid - 1) / grid));
}

constexpr int64_t kPSmemMax = 227 * 1024;

// Deepest ring (up to 8 units per warp) that fits, or 0.
int gemv_p_depth(int M, int64_t K, int64_t N, int rp, bool smem_lut, int num_sms) {
    const int nt = M <= 8 ? 1 : 2;
    const int64_t tiles = (N + 15) / 16;
    const int64_t grid = tiles < num_sms ? tiles : num_sms;
    const int64_t mt = (tiles + grid - 1) / grid;
    if (mt > (1 << 20)) return 0;
    for (int d = 8; d >= 2; --d)
        if (gemv_p_layout(M, K, rp, nt, smem_lut, d, (int)mt).total <= kPSmemMax) return d;
    return 0;
}

// Which GEMV runs: 0 = persistent, with the pair table where a ring of at
// least 3 units still fits, else with the register table; 1 = persistent,
// register table only; 2 = always the per-tile kernel; 3 = as 0 with the
// mixed lookup instead of the pair table.
#ifndef NF4_GEMV_P_MODE
#define NF4_GEMV_P_MODE 0
#endif
#ifndef NF4_GEMV_P_MIN_M
#define NF4_GEMV_P_MIN_M 2
#endif

template <int kMode>
cudaError_t launch_gemv_mode(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                             const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                             void *y, cudaStream_t stream, int num_sms) {
    // Persistent kernel for M >= NF4_GEMV_P_MIN_M when x fits in shared
    // memory: measured on an 11008 x 4096 weight, it matches the per-tile
    // kernel at 2 tokens and is faster from 4 on (8 tokens: 21.8 against
    // 33.5 us, where the per-tile kernel reads x through L1 for every
    // fragment); one token stays on the per-tile kernel.  With LoRA one SM is
    // left to the down-projection that runs alongside (one CTA, whose
    // registers would not fit beside a persistent CTA).
    const int sms = r > 0 && num_sms > 1 ? num_sms - 1 : num_sms;
    if (NF4_GEMV_P_MODE != 2 && K % 256 == 0 && M >= NF4_GEMV_P_MIN_M) {
        constexpr bool kTryPair = NF4_GEMV_P_MODE == 0 || NF4_GEMV_P_MODE == 3;
        constexpr int kPairLut = NF4_GEMV_P_MODE == 3 ? 2 : 1;
        const int d_pair = kTryPair ? gemv_p_depth(M, K, N, rp, true, sms) : 0;
        const int d_reg = gemv_p_depth(M, K, N, rp, false, sms);
        const int nt = M <= 8 ? 1 : 2;
        if (d_pair >= 3 || d_reg >= 2) {
            const bool pair = d_pair >= 3;
            const int d = pair ? d_pair : d_reg;
            const int64_t tiles = (N + 15) / 16, grid = tiles < sms ? tiles : sms;
            const size_t smem = (size_t)gemv_p_layout(M, K, rp, nt, pair, d, (int)((tiles + grid - 1) / grid)).total;
            if (nt == 1)
                return pair ? launch_gemv_p<kMode, 1, kPairLut>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp,
                                                                y, stream, sms, d, smem)
                            : launch_gemv_p<kMode, 1, 0>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y,
                                                         stream, sms, d, smem);
            return pair ? launch_gemv_p<kMode, 2, kPairLut>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y,
                                                            stream, sms, d, smem)
                        : launch_gemv_p<kMode, 2, 0>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, stream,
                                                     sms, d, smem);
        }
    }
    auto *xp = static_cast<const __nv_bfloat16 *>(x);
    auto *bp = static_cast<const __nv_bfloat16 *>(B);
    auto *tp = static_cast<const __nv_bfloat16 *>(t2);
    auto *yp = static_cast<__nv_bfloat16 *>(y);
    // T <= 8: one n8 token tile, 16 weight rows per CTA (more CTAs, better
    // balance); T > 8: two token tiles and 32 rows per CTA, so each x fragment
    // feeds four MMAs and x traffic through L1 stays at 1 byte per weight.
    const int rows_per_cta = M <= 8 ? 16 : 32;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + rows_per_cta - 1) / rows_per_cta));
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.dynamicSmemBytes = kGemvSmemLut ? kPairTableFloat2 * sizeof(float2) : 0;
    if (M <= 8)
        return cudaLaunchKernelEx(&cfg, k_gemv<kMode, 1, 1, kGemvLut>, xp, M, K, N, packed, q8, scales, offset, bp,
                                  r, tp, rp, yp);
    return cudaLaunchKernelEx(&cfg, k_gemv<kMode, 2, 2, kGemvLut>, xp, M, K, N, packed, q8, scales, offset, bp, r,
                              tp, rp, yp);
}

}  // namespace

cudaError_t launch_gemv(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                        const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                        void *y, cudaStream_t stream, int num_sms) {
    if (q8 == nullptr)
        return launch_gemv_mode<2>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, stream, num_sms);
    if (offset == nullptr)
        return launch_gemv_mode<1>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, stream, num_sms);
    return launch_gemv_mode<0>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, stream, num_sms);
}

}  // namespace nf4
