// gemv.cu -- K4: fused NF4-dequantizing linear for small token counts
// (M <= 16), y = x W~^T + [t_hi | t_lo] [B | B]^T.
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

constexpr int kGemvWarps = 4;
#ifndef NF4_GEMV_SMEM_LUT
#define NF4_GEMV_SMEM_LUT 0
#endif
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
template <int kMode, int NT, int MT, bool kSmemLut>
__global__ void __launch_bounds__(kGemvWarps * 32) k_gemv(const __nv_bfloat16 *__restrict__ x, int M, int64_t K,
                                                          int64_t N, const uint8_t *__restrict__ packed,
                                                          const uint8_t *__restrict__ q8,
                                                          const float *__restrict__ scales,
                                                          const float *__restrict__ offset,
                                                          const __nv_bfloat16 *__restrict__ Bl, int r,
                                                          const __nv_bfloat16 *__restrict__ t2, int rp,
                                                          __nv_bfloat16 *__restrict__ y) {
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
        Lut lut[kSmemLut ? 1 : 2 * MT];
        if constexpr (!kSmemLut) {
#pragma unroll
            for (int i = 0; i < 2 * MT; ++i) lut[i] = make_lut(cs[i]);
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
                if constexpr (kSmemLut) {
                    pair_lookup4(tbl_lane, p0, cs[2 * mt], a[0], a[2]);
                    pair_lookup4(tbl_lane, p1, cs[2 * mt + 1], a[1], a[3]);
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

template <int kMode>
cudaError_t launch_gemv_mode(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                             const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                             void *y, cudaStream_t stream) {
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
    cfg.numAttrs = r > 0 ? 1 : 0;  // overlap with the down-projection that precedes it
    cfg.dynamicSmemBytes = kGemvSmemLut ? kPairTableFloat2 * sizeof(float2) : 0;
    if (M <= 8)
        return cudaLaunchKernelEx(&cfg, k_gemv<kMode, 1, 1, kGemvSmemLut>, xp, M, K, N, packed, q8, scales, offset, bp,
                                  r, tp, rp, yp);
    return cudaLaunchKernelEx(&cfg, k_gemv<kMode, 2, 2, kGemvSmemLut>, xp, M, K, N, packed, q8, scales, offset, bp, r,
                              tp, rp, yp);
}

}  // namespace

cudaError_t launch_gemv(const void *x, int M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                        const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                        void *y, cudaStream_t stream) {
    if (q8 == nullptr) return launch_gemv_mode<2>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, stream);
    if (offset == nullptr) return launch_gemv_mode<1>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, stream);
    return launch_gemv_mode<0>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, stream);
}

}  // namespace nf4
