// double_quant.cu -- K2: double quantization of the fp32 block constants.
//
// "QLoRA: Mathematical Foundations ..." (llms.blog), section "Double
// Quantization (DQ)": the first-level constants are grouped in runs of 256,
// each run gets c2 = max |.| and every constant is stored as an 8-bit float
// code of (constant / c2).  Readings (see nf4.h): E4M3 round-to-nearest-even;
// with centring a per-tensor mean mu is subtracted first,
//   mu = RN_f32( RN_f64( S / nblocks ) ),
// S = fixed-order fp64 sum: each run summed sequentially in index order, then
// the run sums combined pairwise level by level, an odd last element carried
// up unchanged.
//
// Kernels
//   k_dq_run_sums    one warp per run: the run's fp64 sum (dq_sum.cuh).  A
//                    tensor sharded over ranks gathers its shards' sums
//                    (nf4_double_quantize_sharded).
//   k_dq_chunks_from_runs
//                    for large tensors only: one thread per chunk of 32
//                    consecutive run sums combines them (a level-5 node of
//                    the pairwise tree).
//   k_dq_quantize    every CTA rebuilds mu from the run sums (folding each
//                    chunk of 32 itself) or from the chunk sums, by the same
//                    tree; then one warp per run computes c2 and the E4M3
//                    codes.
// The pairwise tree restricted to an aligned group of 2^L leaves is the
// perfect tree of that group, and the last partial group follows the same
// level-by-level rule on its own leaves, so splitting the tree at level 5
// reproduces the single-pass order exactly.
//
// Run sums: dq_sum.cuh (in parallel when exact, else sequentially).
#include "dq_sum.cuh"

namespace nf4 {
namespace {

constexpr int kRunsPerChunk = 32;
// Up to this many chunks every CTA of k_dq_quantize folds the run sums into
// chunk sums itself (reading nd doubles, 16 KB at most); above, a separate
// kernel writes the chunk sums once.
constexpr int64_t kDirectChunks = 64;

// Level-by-level pairwise combination of s[0..len) by one thread, in place
// (each level reads s[2j], s[2j+1] before writing s[j], j increasing).
__device__ __forceinline__ double tree_serial(double *s, int64_t len) {
    while (len > 1) {
        int64_t half = len >> 1;
        for (int64_t j = 0; j < half; ++j) s[j] = s[2 * j] + s[2 * j + 1];
        if (len & 1) s[half] = s[len - 1];
        len = half + (len & 1);
    }
    return s[0];
}

// The chunk sum (level-5 node) of runs 32 c .. min(32 c + 32, nd) - 1, by
// one warp (every lane gets it): lane j holds s[j], and each level of the
// pairwise rule (s[j] = s[2j] + s[2j+1], an odd last element carried up) is
// two shuffles.
__device__ __forceinline__ double chunk_sum_warp(const double *__restrict__ run_sums, int64_t nd, int64_t c,
                                                 int lane) {
    int len = (int)(nd - c * kRunsPerChunk < kRunsPerChunk ? nd - c * kRunsPerChunk : kRunsPerChunk);
    double v = lane < len ? run_sums[c * kRunsPerChunk + lane] : 0.0;
    while (len > 1) {  // len is warp-uniform
        const int half = len >> 1;
        const double a = __shfl_sync(0xFFFFFFFFu, v, (2 * lane) & 31);
        const double b = __shfl_sync(0xFFFFFFFFu, v, (2 * lane + 1) & 31);
        const double carry = __shfl_sync(0xFFFFFFFFu, v, len - 1);
        v = lane < half ? a + b : ((len & 1) && lane == half ? carry : 0.0);
        len = half + (len & 1);
    }
    return __shfl_sync(0xFFFFFFFFu, v, 0);
}

// The chunk sum by one thread (level-by-level rule on a local copy).
__device__ __forceinline__ double chunk_sum(const double *__restrict__ run_sums, int64_t nd, int64_t c) {
    double s[kRunsPerChunk];
    int64_t len = nd - c * kRunsPerChunk;
    if (len > kRunsPerChunk) len = kRunsPerChunk;
    for (int64_t j = 0; j < len; ++j) s[j] = run_sums[c * kRunsPerChunk + j];
    return tree_serial(s, len);
}

// Per-run fp64 sums: one warp per run, run_sums[d] for d < ceil(nb / 256).
__global__ void __launch_bounds__(256) k_dq_run_sums(const float *__restrict__ c1, int64_t nb,
                                                      double *__restrict__ run_sums) {
    pdl_wait_then_release();
    const int lane = threadIdx.x & 31;
    const int64_t nd = (nb + kDqBlock - 1) / kDqBlock;
    const int64_t d = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (d >= nd) return;  // whole warps leave together
    const int64_t lo = d * kDqBlock;
    const int64_t cnt = (nb - lo) < kDqBlock ? (nb - lo) : kDqBlock;
    const double sum = run_sum_fp64(c1 + lo, cnt, lane);
    if (lane == 0) run_sums[d] = sum;
}

// Chunk sums of a whole tensor's run sums: one thread per chunk.
__global__ void __launch_bounds__(256) k_dq_chunks_from_runs(const double *__restrict__ run_sums, int64_t nd,
                                                              double *__restrict__ chunk_sums) {
    pdl_wait_then_release();
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nchunks = (nd + kRunsPerChunk - 1) / kRunsPerChunk;
    if (c < nchunks) chunk_sums[c] = chunk_sum(run_sums, nd, c);
}

// Level-by-level pairwise combination of s[0..len) in shared memory (two
// buffers, so no element is overwritten while another thread still reads it).
__device__ double tree_reduce(double *a, double *b, int64_t len) {
    while (len > 1) {
        const int64_t half = len >> 1;
        for (int64_t j = threadIdx.x; j < half; j += blockDim.x) b[j] = a[2 * j] + a[2 * j + 1];
        if ((len & 1) && threadIdx.x == 0) b[half] = a[len - 1];
        __syncthreads();
        double *t = a; a = b; b = t;
        len = half + (len & 1);
    }
    return a[0];
}

// nb constants of c1 are quantized.  With offset non-NULL the mean is
// S / nb_mean, S the tree over the sums: run sums of nd_mean runs when
// sums_are_runs (each CTA folds the chunks itself), else their nchunks chunk
// sums.  nb_mean = nb unless c1 is one shard of a larger tensor.
__global__ void __launch_bounds__(256) k_dq_quantize(const float *__restrict__ c1, int64_t nb,
                                                      const double *__restrict__ sums, int64_t nd_mean,
                                                      int sums_are_runs, int64_t nb_mean,
                                                      uint8_t *__restrict__ codes, float *__restrict__ absmax2,
                                                      float *__restrict__ offset) {
    extern __shared__ double s_tree[];  // 2 * nchunks doubles when centring
    __shared__ float s_mu;
    pdl_wait_then_release();
    if (offset != nullptr) {
        const int64_t nchunks = (nd_mean + kRunsPerChunk - 1) / kRunsPerChunk;
        if (sums_are_runs) {  // one warp per chunk
            const int lane = threadIdx.x & 31;
            for (int64_t j = threadIdx.x >> 5; j < nchunks; j += blockDim.x >> 5) {
                const double cs = chunk_sum_warp(sums, nd_mean, j, lane);
                if (lane == 0) s_tree[j] = cs;
            }
        } else {
            for (int64_t j = threadIdx.x; j < nchunks; j += blockDim.x) s_tree[j] = sums[j];
        }
        __syncthreads();
        double S = tree_reduce(s_tree, s_tree + nchunks, nchunks);
        if (threadIdx.x == 0) {
            float mu = (float)(S / (double)nb_mean);
            s_mu = mu;
            if (blockIdx.x == 0) *offset = mu;
        }
    } else if (threadIdx.x == 0) {
        s_mu = 0.0f;
    }
    __syncthreads();
    const float mu = s_mu;

    const int lane = threadIdx.x & 31;
    const int64_t nd = (nb + kDqBlock - 1) / kDqBlock;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t d = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); d < nd; d += warps_total) {
        const int64_t lo = d * kDqBlock;
        const int64_t cnt = (nb - lo) < kDqBlock ? (nb - lo) : kDqBlock;
        // lane owns constants lo + 8 lane .. lo + 8 lane + 7
        float v[8];
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            int64_t k = 8 * lane + i;
            v[i] = (k < cnt) ? __fsub_rn(__ldg(c1 + lo + k), mu) : 0.0f;
            m = fmaxf(m, fabsf(v[i]));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        const float c2 = m;
        uint8_t q[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) q[i] = (c2 == 0.0f) ? (uint8_t)0 : f32_to_e4m3(__fdiv_rn(v[i], c2));
        if (8 * lane + 8 <= cnt) {
            uint2 pk;
            pk.x = (uint32_t)q[0] | ((uint32_t)q[1] << 8) | ((uint32_t)q[2] << 16) | ((uint32_t)q[3] << 24);
            pk.y = (uint32_t)q[4] | ((uint32_t)q[5] << 8) | ((uint32_t)q[6] << 16) | ((uint32_t)q[7] << 24);
            *reinterpret_cast<uint2 *>(codes + lo + 8 * lane) = pk;
        } else {
            for (int i = 0; i < 8; ++i)
                if (8 * lane + i < cnt) codes[lo + 8 * lane + i] = q[i];
        }
        if (lane == 0) absmax2[d] = c2;
    }
}

}  // namespace

int64_t dq_run_count(int64_t nblocks) { return (nblocks + kDqBlock - 1) / kDqBlock; }
int64_t dq_chunk_count(int64_t nblocks) { return (dq_run_count(nblocks) + kRunsPerChunk - 1) / kRunsPerChunk; }

// Largest chunk count whose tree fits in shared memory (2 buffers of doubles).
int64_t dq_max_chunks() { return (200 * 1024) / (2 * (int64_t)sizeof(double)); }

// Double quantization of nb constants whose runs' fp64 sums (run_sums, of a
// tensor of nb_total constants; nb_total > nb for a shard) are already in
// device memory; chunk_sums: scratch of dq_chunk_count(nb_total) doubles.
// One launch, two for tensors of more than 64 chunks (2048 runs).
cudaError_t launch_dq_from_run_sums(const float *absmax, int64_t nb, const double *run_sums, int64_t nb_total,
                                    uint8_t *codes, float *absmax2, float *offset, double *chunk_sums,
                                    cudaStream_t stream, int num_sms) {
    const int64_t nd_total = dq_run_count(nb_total);
    const int64_t nchunks = dq_chunk_count(nb_total);
    size_t smem = 0;
    const double *sums = run_sums;
    int are_runs = 1;
    if (offset != nullptr) {
        if (nchunks > kDirectChunks) {
            cudaError_t e = launch_pdl(k_dq_chunks_from_runs, dim3((unsigned)((nchunks + 255) / 256)), dim3(256), 0,
                                       stream, 1, run_sums, nd_total, chunk_sums);
            if (e != cudaSuccess) return e;
            sums = chunk_sums;
            are_runs = 0;
        }
        smem = (size_t)(2 * nchunks) * sizeof(double);
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(k_dq_quantize, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
    }
    const int64_t nd = dq_run_count(nb);
    int64_t want = (nd + 7) / 8;
    int64_t cap = (int64_t)num_sms * 4;
    int grid = (int)(want < cap ? want : cap);
    if (grid < 1) grid = 1;  // an empty shard still writes mu
    return launch_pdl(k_dq_quantize, dim3(grid), dim3(256), smem, stream, 1, absmax, nb, sums, nd_total, are_runs,
                      nb_total, codes, absmax2, offset);
}

cudaError_t launch_dq_run_sums(const float *absmax, int64_t nb, double *run_sums, cudaStream_t stream) {
    if (nb == 0) return cudaSuccess;
    const int64_t nd = dq_run_count(nb);
    return launch_pdl(k_dq_run_sums, dim3((unsigned)((nd + 7) / 8)), dim3(256), 0, stream, 1, absmax, nb, run_sums);
}

// nf4_double_quantize: workspace = run sums (nd doubles) then chunk sums.
int64_t dq_workspace_bytes(int64_t nblocks) {
    return (dq_run_count(nblocks) + dq_chunk_count(nblocks)) * (int64_t)sizeof(double);
}

cudaError_t launch_double_quantize(const float *absmax, int64_t nb, uint8_t *codes, float *absmax2,
                                   float *offset, double *workspace, cudaStream_t stream, int num_sms) {
    if (nb == 0) return cudaSuccess;
    if (offset != nullptr) {
        cudaError_t e = launch_dq_run_sums(absmax, nb, workspace, stream);
        if (e != cudaSuccess) return e;
    }
    return launch_dq_from_run_sums(absmax, nb, workspace, nb, codes, absmax2, offset, workspace + dq_run_count(nb),
                                   stream, num_sms);
}

}  // namespace nf4
