// merge.cu -- K7: merge the LoRA adapter into the quantized base and
// requantize, in one pass.
//
// "QLoRA in Production ...", section "Step 4: Merging and Inference": the
// adapter is merged into the quantized base for deployment; "QLoRA: quantising
// the part you are not training", section "What it costs" (item 3): a merge
// into the quantized base has to be requantized.  The pages give no
// arithmetic; the reading (shared with the oracle) is, in binary32,
//   d[n, k]  = fused chain d <- fma(B[n, j], A[j, k], d), j = 0 .. r-1, from +0
//   W'[n, k] = fma(s, d[n, k], w~[n, k]),   w~ = RN(q[code] * c1')
// followed by the blockwise NF4 quantization of W' (c1 = max |W'| per 64-block,
// code = #{i : RN(W' / c1) > t_i}).  The codes depend on every bit of W', so
// the chain runs on the CUDA cores in exactly that order: the tensor cores'
// accumulation order is not specified, and would not reproduce it.
//
// Layout of the work: a CTA owns a tile of 64 rows x 256 columns of W.  A's
// 256 columns (r x 256, fp32) and B's 64 rows (transposed, r x 64, fp32) are
// staged in shared memory once.  Warp w owns rows 8 w .. 8 w + 7 of the tile and lane l
// columns 8 l .. 8 l + 7, so every value of A read from shared memory feeds 8
// rows (64 fma per 2 vector loads and 8 broadcast loads); the 8 lanes
// 8 m .. 8 m + 7 own one 64-block of each row, whose absmax is a 3-step
// shuffle, and the codes come from the quantizer's exact selection.  The merged weight never leaves registers.  packed_out may alias
// packed (every thread reads its 4 code bytes before it writes them), and
// absmax_out may alias fp32 constants (a block's 8 lanes have read its
// constant before the shuffles that precede its write).
#include "mma_util.cuh"
#include "nf4_encode.cuh"

namespace nf4 {
namespace {

constexpr int kMergeCols = 256;
constexpr int kMergeRows = 64;
constexpr int kMergeThreads = 256;
constexpr int kMergeMaxR = 64;
// sB holds B transposed, [j][row] with rows padded to 68 floats: a warp's 8
// rows at one j are two 16-byte broadcast loads (one wavefront each, against
// 8 for 8 scalar loads), and the staging writes, 32 consecutive j of one row,
// hit 8 banks 4 ways.
constexpr int kMergeBStride = kMergeRows + 4;

template <int kMode>
// Two CTAs per SM (128 registers): the epilogue's loads issued before the
// fma chains need ~150 registers, and one CTA per SM was about 40 % slower.
__global__ void __launch_bounds__(kMergeThreads, 2)
    k_merge_requantize(const uint8_t *packed, const uint8_t *__restrict__ q8, const float *scales,
                       const float *__restrict__ offset, int64_t N, int64_t K,
                       const __nv_bfloat16 *__restrict__ A, const __nv_bfloat16 *__restrict__ B, int r, float s,
                       uint8_t *packed_out, float *absmax_out) {
    extern __shared__ float s_dyn[];
    // sA[j][h][l][c] = A[j, k0 + 8 l + 4 h + c]: lane l's two float4 of row j
    // sit 512 bytes apart, so consecutive lanes read consecutive 16 bytes
    float *sA = s_dyn;                      // [r][2][32][4]
    float *sB = s_dyn + r * kMergeCols;     // [r][kMergeBStride], row index fastest
    __shared__ float s_t[16];
    __shared__ uint32_t s_cell[kCellTable];
    __shared__ float s_lv[16];
    const int64_t k0 = (int64_t)blockIdx.x * kMergeCols;
    const int64_t n0 = (int64_t)blockIdx.y * kMergeRows;
    for (int i = threadIdx.x; i < r * kMergeCols; i += kMergeThreads) {
        const int j = i / kMergeCols, col = i % kMergeCols;
        const int l = col >> 3, h = (col >> 2) & 1, c = col & 3;
        const int64_t k = k0 + col;
        sA[j * kMergeCols + h * 128 + l * 4 + c] = k < K ? __bfloat162float(A[(int64_t)j * K + k]) : 0.0f;
    }
    for (int i = threadIdx.x; i < kMergeRows * r; i += kMergeThreads) {
        const int row = i / r, j = i % r;
        const int64_t n = n0 + row;
        sB[j * kMergeBStride + row] = n < N ? __bfloat162float(B[n * r + j]) : 0.0f;
    }
    if (threadIdx.x < 16) s_lv[threadIdx.x] = c_levels[threadIdx.x];
    build_code_tables(s_t, s_cell);  // (synchronises the CTA: sA, sB, s_lv ready too)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;

    // The codes and block-constant operands of this thread's 8 groups are
    // loaded before the fma chains, so their latency is hidden behind them
    // (each group's bytes are still read before this thread writes them).
    const int64_t k = k0 + 8 * lane;
    const bool kvalid = k < K;  // K % 64 == 0: a group of 8 is all in or all out
    uint32_t codes_in[8];
    ScaleRaw sraw[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = n0 + 8 * warp + i;
        const int64_t e = n * K + k;
        if (kvalid && n < N) {
            codes_in[i] = __ldg(reinterpret_cast<const uint32_t *>(packed + (e >> 1)));
            sraw[i] = block_scale_load<kMode>(q8, scales, e >> 6);
        } else {
            codes_in[i] = 0x77777777u;
            sraw[i].q8 = 0u;
            sraw[i].v = 0.0f;
        }
    }

    // d2[i][h] = (d[i][2h], d[i][2h + 1]): row 8 warp + i, columns 8 lane +
    // 2h and 8 lane + 2h + 1 of the tile, as packed fp32 pairs.  Each step of
    // the chain is one fma.rn.f32x2, whose two halves are two independent
    // binary32 fused multiply-adds (each rounded once, to nearest): exactly the
    // scalar chain, at half the instructions.
    uint64_t d2[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int h = 0; h < 4; ++h) d2[i][h] = 0ull;  // (+0, +0)
    const float4 *a_lane = reinterpret_cast<const float4 *>(sA) + lane;
    const float4 *b_warp = reinterpret_cast<const float4 *>(sB + 8 * warp);
#pragma unroll 2
    for (int j = 0; j < r; ++j) {
        const float4 a0 = a_lane[j * 64], a1 = a_lane[j * 64 + 32];
        const float4 b0 = b_warp[j * (kMergeBStride / 4)], b1 = b_warp[j * (kMergeBStride / 4) + 1];
        const uint64_t a2[4] = {pack_f32x2(a0.x, a0.y), pack_f32x2(a0.z, a0.w), pack_f32x2(a1.x, a1.y),
                                pack_f32x2(a1.z, a1.w)};
        const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint64_t bb = pack_f32x2(b[i], b[i]);
#pragma unroll
            for (int h = 0; h < 4; ++h) asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d2[i][h]) : "l"(bb), "l"(a2[h]));
        }
    }
    float d[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int h = 0; h < 4; ++h) asm("mov.b64 {%0, %1}, %2;" : "=f"(d[i][2 * h]), "=f"(d[i][2 * h + 1]) : "l"(d2[i][h]));

#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t n = n0 + 8 * warp + i;
        const bool valid = kvalid && n < N;
        const int64_t e = n * K + k;  // first element of this thread's group
        const float c = valid ? block_scale_finish<kMode>(sraw[i], mu) : 0.0f;
        float w[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            // byte t/2 of the group; element 2j in the high nibble
            const uint32_t code = (codes_in[i] >> (8 * (t >> 1) + ((t & 1) ? 0 : 4))) & 15u;
            const float wt = __fmul_rn(s_lv[code], c);
            w[t] = __fmaf_rn(s, d[i][t], wt);
        }
        float amax = 0.0f;
#pragma unroll
        for (int t = 0; t < 8; ++t) amax = fmaxf(amax, fabsf(w[t]));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, 4));
        if (!valid) continue;
        // codes of RN(W' / c1) (nf4_encode.cuh: division-free, exact)
        const uint32_t out = encode8(w, amax, s_t, s_cell);
        *reinterpret_cast<uint32_t *>(packed_out + (e >> 1)) = out;
        if ((lane & 7) == 0) absmax_out[e >> 6] = amax;
    }
}

template <int kMode>
cudaError_t launch_mode(const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                        int64_t N, int64_t K, const __nv_bfloat16 *A, const __nv_bfloat16 *B, int r, float s,
                        uint8_t *packed_out, float *absmax_out, cudaStream_t stream) {
    const size_t smem = (size_t)(r * kMergeCols + r * kMergeBStride) * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_merge_requantize<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) return e;
    }
    const dim3 grid((unsigned)((K + kMergeCols - 1) / kMergeCols), (unsigned)((N + kMergeRows - 1) / kMergeRows));
    k_merge_requantize<kMode><<<grid, kMergeThreads, smem, stream>>>(packed, q8, scales, offset, N, K, A, B, r, s,
                                                                     packed_out, absmax_out);
    return cudaGetLastError();
}

}  // namespace

int merge_max_rank() { return kMergeMaxR; }

cudaError_t launch_merge_requantize(const uint8_t *packed, const uint8_t *q8, const float *scales,
                                    const float *offset, int64_t N, int64_t K, const void *A, const void *B, int r,
                                    float s, uint8_t *packed_out, float *absmax_out, cudaStream_t stream) {
    if (N <= 0 || K <= 0) return cudaSuccess;
    if ((N + kMergeRows - 1) / kMergeRows > 65535) return cudaErrorInvalidValue;
    auto *ap = static_cast<const __nv_bfloat16 *>(A);
    auto *bp = static_cast<const __nv_bfloat16 *>(B);
    if (q8 == nullptr)
        return launch_mode<2>(packed, q8, scales, offset, N, K, ap, bp, r, s, packed_out, absmax_out, stream);
    if (offset == nullptr)
        return launch_mode<1>(packed, q8, scales, offset, N, K, ap, bp, r, s, packed_out, absmax_out, stream);
    return launch_mode<0>(packed, q8, scales, offset, N, K, ap, bp, r, s, packed_out, absmax_out, stream);
}

}  // namespace nf4
