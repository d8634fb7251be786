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
// 256 columns (r x 256, fp32) and B's 64 rows (transposed, r x 64, each value
// stored twice as an fp32 pair, the broadcast operand of the packed fma) are
// staged in shared memory once, from 16-byte loads of A's and B's rows.
// Warp w owns rows 8 w .. 8 w + 7 of the tile and lane l
// columns 8 l .. 8 l + 7, so every value of A read from shared memory feeds 8
// rows (32 packed fma per 2 + 4 vector loads); the 8 lanes
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
// sB holds B transposed and doubled, [j][row] = (B[row, j], B[row, j]) as fp32
// pairs, rows padded to 136 floats: a warp's 8 rows at one j are four 16-byte
// broadcast loads that give the packed fma its (b, b) operands directly.
constexpr int kMergeBStride = 2 * kMergeRows + 8;

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
    // A: 8 columns (one 16-byte load) per item, written as lane l's two float4
    for (int i = threadIdx.x; i < r * (kMergeCols / 8); i += kMergeThreads) {
        const int j = i >> 5, l = i & 31;  // kMergeCols / 8 == 32
        const int64_t k = k0 + 8 * l;      // K % 64 == 0: 8 columns are all in or all out
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (k < K) u = __ldg(reinterpret_cast<const uint4 *>(A + (int64_t)j * K + k));
        float4 *dst = reinterpret_cast<float4 *>(sA + j * kMergeCols) + l;
        dst[0] = make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                             __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
        dst[32] = make_float4(__uint_as_float(u.z << 16), __uint_as_float(u.z & 0xFFFF0000u),
                              __uint_as_float(u.w << 16), __uint_as_float(u.w & 0xFFFF0000u));
    }
    // B: 8 consecutive j of one row (one 16-byte load) per item when r % 8 ==
    // 0 (rows 16-byte aligned), else one value per item; each value written
    // as the pair (b, b)
    if ((r & 7) != 0) {
        for (int i = threadIdx.x; i < kMergeRows * r; i += kMergeThreads) {
            const int row = i % kMergeRows, j = i / kMergeRows;
            const int64_t n = n0 + row;
            const float b = n < N ? __bfloat162float(B[n * r + j]) : 0.0f;
            *reinterpret_cast<float2 *>(sB + j * kMergeBStride + 2 * row) = make_float2(b, b);
        }
    }
    for (int i = threadIdx.x; (r & 7) == 0 && i < kMergeRows * (r / 8); i += kMergeThreads) {
        const int row = i % kMergeRows, j0 = (i / kMergeRows) * 8;
        const int64_t n = n0 + row;
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (n < N) u = __ldg(reinterpret_cast<const uint4 *>(B + n * r + j0));
        const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const float b = __uint_as_float((t & 1) ? (w4[t >> 1] & 0xFFFF0000u) : (w4[t >> 1] << 16));
            *reinterpret_cast<float2 *>(sB + (j0 + t) * kMergeBStride + 2 * row) = make_float2(b, b);
        }
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
    const ulonglong2 *a_lane = reinterpret_cast<const ulonglong2 *>(sA) + lane;
    const ulonglong2 *b_warp = reinterpret_cast<const ulonglong2 *>(sB + 16 * warp);
#pragma unroll 2
    for (int j = 0; j < r; ++j) {
        // (A[j, 8l + 2h], A[j, 8l + 2h + 1]) pairs and (B[8w + i, j]) x 2
        const ulonglong2 a01 = a_lane[j * 64], a23 = a_lane[j * 64 + 32];
        const uint64_t a2[4] = {a01.x, a01.y, a23.x, a23.y};
        uint64_t bb[8];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const ulonglong2 p = b_warp[j * (kMergeBStride / 4) + m];
            bb[2 * m] = p.x;
            bb[2 * m + 1] = p.y;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int h = 0; h < 4; ++h) asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d2[i][h]) : "l"(bb[i]), "l"(a2[h]));
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
