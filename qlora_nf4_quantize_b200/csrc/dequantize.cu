// dequantize.cu -- K3: NF4 dequantization to fp32 or bf16.
//
// "QLoRA: Mathematical Foundations ..." (llms.blog), section "Block-Wise
// Quantization Mechanics", dequantization equation: w~ = c1 * q[code], one
// binary32 multiply; c1 is the block constant reconstructed from the double
// quantization state (nf4_device.cuh, block_scale).  bf16 output rounds the
// binary32 value to nearest even.
//
// HBM-bound streaming kernel: a lane owns 8 consecutive elements per step
// (4 packed bytes: one 32-bit load, a warp reads 128 contiguous bytes), looks
// the 8 codes up in a 16-entry shared-memory copy of the table (16 distinct
// words in 16 banks: conflict-free for any code pattern) and writes 32 bytes
// (fp32) or 16 bytes (bf16) with 128-bit stores.  The 8 lanes that share a
// 64-block read the same scale byte (one broadcast request).
#include "nf4_device.cuh"

namespace nf4 {
namespace {

constexpr int kDeqThreads = 256;

template <int kMode, bool kBf16Out>
__global__ void __launch_bounds__(kDeqThreads) k_dequantize(const uint8_t *__restrict__ packed,
                                                             const uint8_t *__restrict__ q8,
                                                             const float *__restrict__ scales,
                                                             const float *__restrict__ offset, int64_t n,
                                                             void *__restrict__ out) {
    __shared__ float s_q[16];
    if (threadIdx.x < 16) s_q[threadIdx.x] = c_levels[threadIdx.x];
    __syncthreads();
    const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
    const int64_t ngroups = (n + 7) >> 3;
    for (int64_t g = (int64_t)blockIdx.x * kDeqThreads + threadIdx.x; g < ngroups;
         g += (int64_t)gridDim.x * kDeqThreads) {
        const int64_t e0 = g << 3;
        const float c = block_scale<kMode>(q8, scales, mu, e0 >> 6);
        if (e0 + 8 <= n) {
            const uint32_t p = __ldg(reinterpret_cast<const uint32_t *>(packed) + g);
            float v[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t byte = (p >> (8 * j)) & 0xFFu;
                v[2 * j] = __fmul_rn(s_q[byte >> 4], c);       // element 2j: high nibble
                v[2 * j + 1] = __fmul_rn(s_q[byte & 15u], c);  // element 2j+1: low nibble
            }
            if constexpr (kBf16Out) {
                uint4 o;
                o.x = pack_bf16x2(v[0], v[1]);
                o.y = pack_bf16x2(v[2], v[3]);
                o.z = pack_bf16x2(v[4], v[5]);
                o.w = pack_bf16x2(v[6], v[7]);
                reinterpret_cast<uint4 *>(out)[g] = o;
            } else {
                float4 *dst = reinterpret_cast<float4 *>(out) + 2 * g;
                dst[0] = make_float4(v[0], v[1], v[2], v[3]);
                dst[1] = make_float4(v[4], v[5], v[6], v[7]);
            }
        } else {
            for (int64_t e = e0; e < n; ++e) {
                const uint32_t byte = packed[e >> 1];
                const uint32_t code = (e & 1) ? (byte & 15u) : (byte >> 4);
                const float v = __fmul_rn(s_q[code], c);
                if constexpr (kBf16Out) reinterpret_cast<__nv_bfloat16 *>(out)[e] = __float2bfloat16_rn(v);
                else reinterpret_cast<float *>(out)[e] = v;
            }
        }
    }
}

template <int kMode>
cudaError_t launch_mode(const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                        int64_t n, void *out, bool bf16, int grid, cudaStream_t stream) {
    if (bf16) k_dequantize<kMode, true><<<grid, kDeqThreads, 0, stream>>>(packed, q8, scales, offset, n, out);
    else k_dequantize<kMode, false><<<grid, kDeqThreads, 0, stream>>>(packed, q8, scales, offset, n, out);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_dequantize(const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                              int64_t n, void *out, bool bf16, cudaStream_t stream, int num_sms) {
    if (n == 0) return cudaSuccess;
    int64_t ngroups = (n + 7) / 8;
    int64_t want = (ngroups + kDeqThreads - 1) / kDeqThreads;
    int64_t cap = (int64_t)num_sms * 8;
    int grid = (int)(want < cap ? want : cap);
    if (q8 == nullptr) return launch_mode<2>(packed, q8, scales, offset, n, out, bf16, grid, stream);
    if (offset == nullptr) return launch_mode<1>(packed, q8, scales, offset, n, out, bf16, grid, stream);
    return launch_mode<0>(packed, q8, scales, offset, n, out, bf16, grid, stream);
}

}  // namespace nf4
