// nf4_device.cuh -- device-side definitions shared by the NF4 kernels.
//
// The NF4 table is the list printed on "QLoRA: Mathematical Foundations of
// 4-Bit NormalFloat Quantization, Double Quantization, and Paged Optimizers"
// (llms.blog), section "4-Bit NormalFloat (NF4): Information-Theoretic
// Quantile Quantization"; every printed decimal is an exact binary32 value.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace nf4 {

constexpr int kBlock = 64;      // first-level block ("B_1 = 64")
constexpr int kDqBlock = 256;   // second-level block ("B_2 = 256")

// Host copy (used to fill device tables and by nf4_codebook()).
static const float kLevelsHost[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
    0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};

// Device copy in constant memory (broadcast reads only; kernels that index it
// per element first copy it to shared memory).
static __constant__ float c_levels[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
    0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};

// OCP FP8 E4M3 byte -> fp32 (exact: every E4M3 value is an fp16 value).
__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
    return __half2float(__half(h));
}

// fp32 -> E4M3, round to nearest even, saturating to +-448.
__device__ __forceinline__ uint8_t f32_to_e4m3(float y) {
    return (uint8_t)__nv_cvt_float_to_fp8(y, __NV_SATFINITE, __NV_E4M3);
}

// Reconstructed first-level constant of block b (see nf4_dequantize in nf4.h).
//   kMode 0: double quantization with centring  c = fma(E4M3(q8), c2, mu)
//   kMode 1: double quantization, no centring   c = E4M3(q8) * c2
//   kMode 2: no double quantization            c = scales[b] (fp32 c1)
template <int kMode>
__device__ __forceinline__ float block_scale(const uint8_t *__restrict__ q8, const float *__restrict__ scales,
                                             float mu, int64_t b) {
    if constexpr (kMode == 2) {
        return __ldg(scales + b);
    } else {
        float d = e4m3_to_f32(__ldg(q8 + b));
        float c2 = __ldg(scales + (b >> 8));
        if constexpr (kMode == 0) return __fmaf_rn(d, c2, mu);
        else return __fmul_rn(d, c2);
    }
}

// Raw operands of a block constant, loaded ahead of use so that the loads
// overlap other work; block_scale_finish() turns them into c1'.
struct ScaleRaw {
    uint32_t q8;  // E4M3 code (kMode 0, 1)
    float v;      // c2 (kMode 0, 1) or the fp32 c1 itself (kMode 2)
};

template <int kMode>
__device__ __forceinline__ ScaleRaw block_scale_load(const uint8_t *__restrict__ q8, const float *__restrict__ scales,
                                                     int64_t b) {
    ScaleRaw r;
    if constexpr (kMode == 2) {
        r.q8 = 0;
        r.v = __ldg(scales + b);
    } else {
        r.q8 = __ldg(q8 + b);
        r.v = __ldg(scales + (b >> 8));
    }
    return r;
}

template <int kMode>
__device__ __forceinline__ float block_scale_finish(const ScaleRaw &r, float mu) {
    if constexpr (kMode == 2) {
        return r.v;
    } else {
        const float d = e4m3_to_f32((uint8_t)r.q8);
        if constexpr (kMode == 0) return __fmaf_rn(d, r.v, mu);
        else return __fmul_rn(d, r.v);
    }
}

// Code selection (section "Block-Wise Quantization Mechanics"): the code of a
// normalised value x is the arg-min of |x - q_i| with ties to the lower
// index, i.e. #{i : x > t_i} with t_i = RD_f32((q_i + q_{i+1}) / 2), the exact
// midpoint rounded down.  fill_thresholds writes t_0..t_14 (call from one
// thread or with a barrier after).
__device__ __forceinline__ void fill_thresholds(float *s_t) {
    for (int i = threadIdx.x; i < 15; i += blockDim.x) {
        const double m = ((double)c_levels[i] + (double)c_levels[i + 1]) * 0.5;  // exact in binary64
        s_t[i] = __double2float_rd(m);
    }
}

__device__ __forceinline__ int code_of_quotient(float x, const float *s_t) {
    int c = 0;
#pragma unroll
    for (int i = 0; i < 15; ++i) c += (x > s_t[i]) ? 1 : 0;
    return c;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
    return *reinterpret_cast<uint32_t *>(&v);
}

// Programmatic dependent launch, used by every kernel of the library: a
// kernel launched with launch_pdl() first waits for the grid before it in the
// stream (completion and memory visibility; immediate if that grid did not
// release it early), then releases the grid after it, which may then be
// scheduled while this one still runs and waits in turn before touching
// memory.  Only launch latency overlaps; data order is the stream's order.
__device__ __forceinline__ void pdl_wait_then_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// cudaLaunchKernelEx with the programmatic-serialization attribute (and a
// cluster size when cluster_x > 1).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              unsigned cluster_x, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int na = 1;
    if (cluster_x > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster_x;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        na = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = na;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace nf4
