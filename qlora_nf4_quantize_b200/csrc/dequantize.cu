// dequantize.cu -- K3: NF4 dequantization to fp32 or bf16.
//
// "QLoRA: Mathematical Foundations ..." (llms.blog), section "Block-Wise
// Quantization Mechanics", dequantization equation: w~ = c1 * q[code], one
// binary32 multiply; c1 is the block constant reconstructed from the double
// quantization state (nf4_device.cuh, block_scale).  bf16 output rounds the
// binary32 value to nearest even.
//
// HBM-bound streaming kernel.  A warp handles kSeg * 256 consecutive elements
// per iteration as kSeg segments of 256.  bf16 output: in segment j lane l
// owns the 8 elements starting at 256 j + 8 l, i.e. 4 packed bytes (one
// 32-bit load; the warp's load is 128 contiguous bytes) and 16 output bytes
// (one 128-bit store; the warp's store is 512 contiguous bytes).  fp32
// output: lane l owns elements 256 j + 4 l .. + 3 and 256 j + 128 + 4 l .. + 3
// (two 16-bit loads), so each of its two 128-bit stores is 512 contiguous
// bytes per warp; 8 consecutive elements per lane would make every store
// instruction write every other 16 bytes (4096 x 4096: 19.3 -> 14.7 us).  All kSeg loads of
// a lane (codes and block constants) are issued before any arithmetic; up to
// 8 CTAs of 256 threads per SM are resident, and the grid may hold more (see
// launch_mode for the shape).  Eight segments per iteration (a 4096 x 4096
// weight read in one round trip per warp) measured slower than four.
// Codes are looked up in a 16-entry shared-memory copy of the table (16
// distinct words in 16 banks: conflict-free for any code pattern).
#include "nf4_device.cuh"

namespace nf4 {
namespace {

constexpr int kDeqThreads = 256;

// 8 consecutive bf16 outputs as one 16-byte store.
__device__ __forceinline__ void store8_bf16(void *out, int64_t e0, const float v[8]) {
    uint4 o;
    o.x = pack_bf16x2(v[0], v[1]);
    o.y = pack_bf16x2(v[2], v[3]);
    o.z = pack_bf16x2(v[4], v[5]);
    o.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(out) + e0) = o;
}

template <int kMode, bool kBf16Out, int kSeg>
__global__ void __launch_bounds__(kDeqThreads, 2048 / kDeqThreads) k_dequantize(const uint8_t *__restrict__ packed,
                                                             const uint8_t *__restrict__ q8,
                                                             const float *__restrict__ scales,
                                                             const float *__restrict__ offset, int64_t n,
                                                             void *__restrict__ out) {
    constexpr int kWarpElems = kSeg * 256;  // elements per warp per iteration
    static_assert(16384 % kWarpElems == 0, "a warp iteration stays in one group of 256 blocks");
    __shared__ float s_q[16];
    pdl_wait_then_release();
    if (threadIdx.x < 16) s_q[threadIdx.x] = c_levels[threadIdx.x];
    __syncthreads();
    const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (kDeqThreads / 32);
    const int64_t nfull = n / kWarpElems;  // warp iterations with no tail
    for (int64_t c = (int64_t)blockIdx.x * (kDeqThreads / 32) + (threadIdx.x >> 5); c < nfull && !kBf16Out;
         c += warps) {
        // fp32 output: in segment j lane l owns elements 4l..4l+3 and
        // 128+4l..128+4l+3, so each 16-byte store of the warp covers 512
        // contiguous bytes (with 8 consecutive elements per lane a store
        // instruction would write every other 16 bytes)
        const int64_t seg0 = c * kWarpElems;
        uint32_t ph[kSeg][2];
        ScaleRaw sr[kSeg][2];
#pragma unroll
        for (int j = 0; j < kSeg; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h)
                ph[j][h] = __ldg(reinterpret_cast<const uint16_t *>(packed) + ((seg0 + 256 * j + 128 * h + 4 * lane) >> 2));
        const float c2 = (kMode == 2) ? 0.0f : __ldg(scales + (seg0 >> 14));
#pragma unroll
        for (int j = 0; j < kSeg; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t blk = (seg0 + 256 * j + 128 * h + 4 * lane) >> 6;
                if constexpr (kMode == 2) {
                    sr[j][h].v = __ldg(scales + blk);
                } else {
                    sr[j][h].q8 = __ldg(q8 + blk);
                    sr[j][h].v = c2;
                }
            }
#pragma unroll
        for (int j = 0; j < kSeg; ++j)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const float scj = block_scale_finish<kMode>(sr[j][h], mu);
                const uint32_t w = ph[j][h];  // byte 0 = elements 0, 1; byte 1 = elements 2, 3
                float4 v;
                v.x = __fmul_rn(s_q[(w >> 4) & 15u], scj);
                v.y = __fmul_rn(s_q[w & 15u], scj);
                v.z = __fmul_rn(s_q[(w >> 12) & 15u], scj);
                v.w = __fmul_rn(s_q[(w >> 8) & 15u], scj);
                *reinterpret_cast<float4 *>(static_cast<float *>(out) + seg0 + 256 * j + 128 * h + 4 * lane) = v;
            }
    }
    for (int64_t c = (int64_t)blockIdx.x * (kDeqThreads / 32) + (threadIdx.x >> 5); c < nfull && kBf16Out;
         c += warps) {
        const int64_t base = c * kWarpElems + 8 * lane;
        uint32_t p[kSeg];
        ScaleRaw sr[kSeg];
#pragma unroll
        for (int j = 0; j < kSeg; ++j) p[j] = __ldg(reinterpret_cast<const uint32_t *>(packed) + ((base + 256 * j) >> 3));
        if constexpr (kMode == 2) {
#pragma unroll
            for (int j = 0; j < kSeg; ++j) sr[j].v = __ldg(scales + ((base + 256 * j) >> 6));
        } else {
            // the iteration's kSeg * 256 elements lie in one group of 256
            // blocks (kSeg * 256 divides 16384): one second-level constant
            const float c2 = __ldg(scales + ((c * kWarpElems) >> 14));
#pragma unroll
            for (int j = 0; j < kSeg; ++j) {
                sr[j].q8 = __ldg(q8 + ((base + 256 * j) >> 6));
                sr[j].v = c2;
            }
        }
#pragma unroll
        for (int j = 0; j < kSeg; ++j) {
            const float scj = block_scale_finish<kMode>(sr[j], mu);
            float v[8];
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint32_t byte = (p[j] >> (8 * b)) & 0xFFu;
                v[2 * b] = __fmul_rn(s_q[byte >> 4], scj);       // element 2b: high nibble
                v[2 * b + 1] = __fmul_rn(s_q[byte & 15u], scj);  // element 2b+1: low nibble
            }
            store8_bf16(out, base + 256 * j, v);
        }
    }
    // tail: elements [nfull * kWarpElems, n), one element per thread
    const int64_t tail0 = nfull * kWarpElems;
    for (int64_t e = tail0 + (int64_t)blockIdx.x * kDeqThreads + threadIdx.x; e < n;
         e += (int64_t)gridDim.x * kDeqThreads) {
        const float c1 = block_scale<kMode>(q8, scales, mu, e >> 6);
        const uint32_t byte = packed[e >> 1];
        const uint32_t code = (e & 1) ? (byte & 15u) : (byte >> 4);
        const float v = __fmul_rn(s_q[code], c1);
        if constexpr (kBf16Out) reinterpret_cast<__nv_bfloat16 *>(out)[e] = __float2bfloat16_rn(v);
        else reinterpret_cast<float *>(out)[e] = v;
    }
}

template <int kMode, int kSeg>
cudaError_t launch_seg(const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset, int64_t n,
                       void *out, bool bf16, int ctas_per_sm, int num_sms, cudaStream_t stream) {
    const int64_t witers = (n + kSeg * 256 - 1) / (kSeg * 256);
    const int64_t want = (witers + (kDeqThreads / 32) - 1) / (kDeqThreads / 32);
    const int64_t cap = (int64_t)num_sms * ctas_per_sm;
    const int grid = (int)(want < cap ? want : cap);
    if (bf16)
        return launch_pdl(k_dequantize<kMode, true, kSeg>, dim3(grid), dim3(kDeqThreads), 0, stream, 1, packed, q8,
                          scales, offset, n, out);
    return launch_pdl(k_dequantize<kMode, false, kSeg>, dim3(grid), dim3(kDeqThreads), 0, stream, 1, packed, q8,
                      scales, offset, n, out);
}

// Launch shape, measured on B200 (4096 x 4096 and 14336 x 4096 weights): a
// bf16 output of up to 2^25 elements runs 2 segments per lane and iteration
// with the grid capped at 16 CTAs per SM (about 1.7 iterations per warp, so
// CTAs that finish early are followed by the rest); larger outputs and fp32
// runs 4 segments with the grid capped at 32 CTAs per SM.  Both shapes beat
// 4 segments at 8 CTAs per SM (a single resident wave) by 5-11 %.
template <int kMode>
cudaError_t launch_mode(const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                        int64_t n, void *out, bool bf16, int num_sms, cudaStream_t stream) {
    if (bf16 && n <= (int64_t(1) << 25))
        return launch_seg<kMode, 2>(packed, q8, scales, offset, n, out, bf16, 16, num_sms, stream);
    return launch_seg<kMode, 4>(packed, q8, scales, offset, n, out, bf16, 32, num_sms, stream);
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                              int64_t n, void *out, bool bf16, cudaStream_t stream, int num_sms) {
    if (n == 0) return cudaSuccess;
    if (q8 == nullptr) return launch_mode<2>(packed, q8, scales, offset, n, out, bf16, num_sms, stream);
    if (offset == nullptr) return launch_mode<1>(packed, q8, scales, offset, n, out, bf16, num_sms, stream);
    return launch_mode<0>(packed, q8, scales, offset, n, out, bf16, num_sms, stream);
}

}  // namespace nf4
