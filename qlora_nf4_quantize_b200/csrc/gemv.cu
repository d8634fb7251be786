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
//   - A CTA (4 warps) owns a tile of 32 weight rows; the warps split K in
//     super-steps of 256 columns (warp w takes super-steps w, w+4, ...) and
//     their partial sums are added in shared memory in warp order.
//   - Each warp runs m16n8k16 tensor-core MMAs with the weight as the A
//     operand (two m16 tiles) and x as the B operand (one n8 tile per 8
//     tokens).  Within a super-step the K index is permuted so that the four
//     A-fragment columns a lane owns at MMA step s (2t, 2t+1, 2t+8, 2t+9) are
//     elements 4s..4s+3 of 64-block t of its rows; the x fragment uses the
//     same permutation (one 8-byte load of x[token, 64 t + 4 s ...]).  So a
//     lane dequantizes whole 64-blocks: one scale and one register lookup
//     table (mma_util.cuh, make_lut) per block, then 3 byte permutes per
//     weight and no shared memory.
//   - The LoRA term is a K-extension of 2r columns after the reduction, and
//     the CTA writes its 32 x M outputs.
#include "mma_util.cuh"

namespace nf4 {
namespace {

constexpr int kGemvWarps = 4;
constexpr int kRowsPerCta = 32;

// 32 packed bytes (64 codes) of row `row`, 64-block `bk`, or all-zero-code
// words (0x77) outside the matrix.
__device__ __forceinline__ void load_block_codes(const uint8_t *__restrict__ packed, int64_t row, int64_t K,
                                                 int64_t bk, bool valid, uint32_t w[8]) {
    if (valid) {
        const uint4 *p = reinterpret_cast<const uint4 *>(packed + row * (K >> 1) + bk * 32);
        uint4 u0 = __ldg(p), u1 = __ldg(p + 1);
        w[0] = u0.x; w[1] = u0.y; w[2] = u0.z; w[3] = u0.w;
        w[4] = u1.x; w[5] = u1.y; w[6] = u1.z; w[7] = u1.w;
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = 0x77777777u;
    }
}

template <int kMode, int NT>
__global__ void __launch_bounds__(kGemvWarps * 32) k_gemv(const __nv_bfloat16 *__restrict__ x, int M, int64_t K,
                                                          int64_t N, const uint8_t *__restrict__ packed,
                                                          const uint8_t *__restrict__ q8,
                                                          const float *__restrict__ scales,
                                                          const float *__restrict__ offset,
                                                          const __nv_bfloat16 *__restrict__ Bl, int r,
                                                          const __nv_bfloat16 *__restrict__ t2, int rp,
                                                          __nv_bfloat16 *__restrict__ y) {
    __shared__ float s_part[kGemvWarps][2][NT][4][32];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int64_t n0 = (int64_t)blockIdx.x * kRowsPerCta;
    const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
    const int64_t kblocks = K >> 6;             // 64-blocks per row
    const int64_t nsuper = (kblocks + 3) >> 2;  // super-steps of 4 blocks

    // rows owned by this lane: n0 + g + 8 i, i = 0..3 (m-tile 0: i = 0, 1; m-tile 1: i = 2, 3)
    int64_t row[4];
    bool rvalid[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
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

    float acc[2][NT][4];
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0.0f;

    for (int64_t ss = warp; ss < nsuper; ss += kGemvWarps) {
        const int64_t bk = ss * 4 + tq;  // this lane's 64-block along K
        const bool kvalid = bk < kblocks;
        uint32_t cw[4][8];
        Lut lut[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const bool v = rvalid[i] && kvalid;
            load_block_codes(packed, row[i], K, bk, v, cw[i]);
            const float c = v ? block_scale<kMode>(q8, scales, mu, row[i] * kblocks + bk) : 0.0f;
            lut[i] = make_lut(c);
        }
        const int64_t kx = bk * 64;  // x column of element 0 of this block (in 4-element units below)
#pragma unroll
        for (int s = 0; s < 16; ++s) {
            uint2 xb[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) xb[nt] = (tvalid[nt] && kvalid) ? __ldg(xrow[nt] + ((kx >> 2) + s)) : make_uint2(0u, 0u);
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                uint32_t a[4];
                const uint32_t p0 = cw[2 * mt][s >> 1] >> ((s & 1) * 16);
                const uint32_t p1 = cw[2 * mt + 1][s >> 1] >> ((s & 1) * 16);
                lut_lookup4(lut[2 * mt], p0, a[0], a[2]);
                lut_lookup4(lut[2 * mt + 1], p1, a[1], a[3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16_16816(acc[mt][nt], a, xb[nt].x, xb[nt].y);
            }
        }
    }

#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) s_part[warp][mt][nt][i][lane] = acc[mt][nt][i];
    __syncthreads();
    if (warp != 0) return;
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
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
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                uint32_t a[4];
                const int64_t ra = row[2 * mt], rb = row[2 * mt + 1];
                const uint32_t *ba = reinterpret_cast<const uint32_t *>(Bl + (rvalid[2 * mt] ? ra : 0) * r);
                const uint32_t *bb = reinterpret_cast<const uint32_t *>(Bl + (rvalid[2 * mt + 1] ? rb : 0) * r);
                const int w0 = (j0 + 2 * tq) >> 1;
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
    for (int mt = 0; mt < 2; ++mt)
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
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((N + kRowsPerCta - 1) / kRowsPerCta));
    cfg.blockDim = dim3(kGemvWarps * 32);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = r > 0 ? 1 : 0;  // overlap with the down-projection that precedes it
    if (M <= 8)
        return cudaLaunchKernelEx(&cfg, k_gemv<kMode, 1>, xp, M, K, N, packed, q8, scales, offset, bp, r, tp, rp, yp);
    return cudaLaunchKernelEx(&cfg, k_gemv<kMode, 2>, xp, M, K, N, packed, q8, scales, offset, bp, r, tp, rp, yp);
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
