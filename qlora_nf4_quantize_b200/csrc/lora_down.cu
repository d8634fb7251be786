// lora_down.cu -- K6: the LoRA down-projection t = s * x A^T of the forward
// pass ("QLoRA: Mathematical Foundations ...", section "Forward Pass
// Computation": the (alpha / r)(X L1) term, L1 = A^T), computed once per call
// before the fused linear.
//
// Output (the caller's workspace): t2[M, RP] bf16 with RP = round_up(2r, 64),
//   t2[m, j]     = t_hi = RNE_bf16(v),          j < r
//   t2[m, r + j] = t_lo = RNE_bf16(v - t_hi),    j < r
//   t2[m, j]     = 0,                            2r <= j < RP
// with v = s * sum_k x[m, k] A[j, k] accumulated in fp32.  t_hi + t_lo keeps
// about 16 significant bits of v, so the low-rank term is not limited by
// bf16 rounding of t; the consumers multiply [t_hi | t_lo] by [B | B].
//
// Layout of the work: a CTA owns 16 rows of x; its 16 warps split K (warp w
// takes k16-steps w, w+16, ...), each warp runs m16n8k16 MMAs over all r
// columns, and the 16 partial tiles are summed in shared memory in warp
// order.  For decode-size M the whole projection is one CTA whose warps each
// issue all their loads up front, so its latency is a few memory round trips.
// The kernel triggers programmatic dependent launch at entry: the fused
// linear that follows starts streaming the weight at once and waits for t
// only where it reads it (griddepcontrol.wait).
#include "mma_util.cuh"

namespace nf4 {
namespace {

constexpr int kDownWarps = 16;

template <int kR>
__global__ void __launch_bounds__(kDownWarps * 32) k_lora_down(const __nv_bfloat16 *__restrict__ x,
                                                               const __nv_bfloat16 *__restrict__ A, int64_t M,
                                                               int64_t K, float s, __nv_bfloat16 *__restrict__ t2,
                                                               int rp) {
    constexpr int NT = kR / 8;  // n8 tiles
    extern __shared__ float s_part_raw[];  // [kDownWarps][NT][4][32]
    auto s_part = reinterpret_cast<float (*)[NT][4][32]>(s_part_raw);
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int64_t m0 = (int64_t)blockIdx.x * 16;
    const int64_t ra = m0 + g, rb = m0 + g + 8;
    const bool va = ra < M, vb = rb < M;
    const uint32_t *xa = reinterpret_cast<const uint32_t *>(x + (va ? ra : 0) * K);
    const uint32_t *xb = reinterpret_cast<const uint32_t *>(x + (vb ? rb : 0) * K);

    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

    const int64_t ksteps = K / 16;
#pragma unroll 4
    for (int64_t kk = warp; kk < ksteps; kk += kDownWarps) {
        const int64_t kw = (kk * 16 + 2 * tq) >> 1;  // 32-bit word index of column 16 kk + 2 tq
        uint32_t a[4];
        a[0] = va ? __ldg(xa + kw) : 0u;
        a[1] = vb ? __ldg(xb + kw) : 0u;
        a[2] = va ? __ldg(xa + kw + 4) : 0u;
        a[3] = vb ? __ldg(xb + kw + 4) : 0u;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const uint32_t *ar = reinterpret_cast<const uint32_t *>(A + (int64_t)(nt * 8 + g) * K);
            mma_bf16_16816(acc[nt], a, __ldg(ar + kw), __ldg(ar + kw + 4));
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) s_part[warp][nt][i][lane] = acc[nt][i];
    __syncthreads();
    // 16 rows x kR columns = 16 kR outputs, shared by all threads
    for (int o = threadIdx.x; o < NT * 4 * 32; o += kDownWarps * 32) {
        const int nt = o / 128, i = (o / 32) & 3, ln = o & 31;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kDownWarps; ++w) v += s_part[w][nt][i][ln];
        v *= s;
        const int row = (ln >> 2) + ((i & 2) ? 8 : 0);
        const int col = nt * 8 + 2 * (ln & 3) + (i & 1);
        const int64_t m = m0 + row;
        if (m < M) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
            t2[m * rp + col] = hi;
            t2[m * rp + kR + col] = lo;
        }
    }
    // zero padding columns [2r, rp)
    for (int o = threadIdx.x; o < 16 * (rp - 2 * kR); o += kDownWarps * 32) {
        const int row = o / (rp - 2 * kR), col = 2 * kR + o % (rp - 2 * kR);
        if (m0 + row < M) t2[(m0 + row) * rp + col] = __float2bfloat16_rn(0.0f);
    }
}

template <int kR>
cudaError_t launch_down(unsigned grid, size_t smem, cudaStream_t stream, const __nv_bfloat16 *x,
                        const __nv_bfloat16 *A, int64_t M, int64_t K, float s, __nv_bfloat16 *t2, int rp) {
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_lora_down<kR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_lora_down<kR><<<grid, kDownWarps * 32, smem, stream>>>(x, A, M, K, s, t2, rp);
    return cudaSuccess;
}

}  // namespace

int lora_rp(int r) { return ((2 * r + 63) / 64) * 64; }

cudaError_t launch_lora_down(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2,
                             cudaStream_t stream) {
    const unsigned grid = (unsigned)((M + 15) / 16);
    const int rp = lora_rp(r);
    const size_t smem = (size_t)kDownWarps * (r / 8) * 4 * 32 * sizeof(float);
    auto *xp = static_cast<const __nv_bfloat16 *>(x);
    auto *ap = static_cast<const __nv_bfloat16 *>(A);
    auto *tp = static_cast<__nv_bfloat16 *>(t2);
    cudaError_t e = cudaSuccess;
    switch (r) {
        case 16: e = launch_down<16>(grid, smem, stream, xp, ap, M, K, s, tp, rp); break;
        case 32: e = launch_down<32>(grid, smem, stream, xp, ap, M, K, s, tp, rp); break;
        case 64: e = launch_down<64>(grid, smem, stream, xp, ap, M, K, s, tp, rp); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace nf4
