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
// Layout of the work (M <= 16, one m16 tile of x rows): one thread-block
// cluster of kDownCtas CTAs x 16 warps splits K (global warp w = rank * 16 +
// warp takes k16-steps w, w + 128, ...); each warp runs m16n8k16 MMAs over all
// r columns and issues its loads up front.  Each CTA sums its 16 warps'
// partial tiles in shared memory in warp order; then every CTA takes a slice
// of the 16 x r outputs and sums the CTAs' partials in rank order through
// distributed shared memory, so the result is independent of timing.  The
// kernel releases the fused linear that follows (programmatic dependent
// launch) as soon as its own predecessor has completed: the linear starts
// streaming the weight at once and waits for t only where it reads it.  For a
// linear split over the SMs (9 to 16 tokens) it also zeroes that linear's
// per-tile arrival counts in the caller's workspace.
#include <cooperative_groups.h>

#include "mma_util.cuh"

namespace nf4 {
namespace {

namespace cg = cooperative_groups;

constexpr int kDownWarps = 16;
constexpr int kDownCtas = 8;  // cluster size (portable maximum)

template <int kR>
__global__ void __launch_bounds__(kDownWarps * 32) k_lora_down(const __nv_bfloat16 *__restrict__ x,
                                                               const __nv_bfloat16 *__restrict__ A, int64_t M,
                                                               int64_t K, float s, __nv_bfloat16 *__restrict__ t2,
                                                               int rp, unsigned *__restrict__ counts, int ncounts) {
    constexpr int NT = kR / 8;  // n8 tiles
    extern __shared__ float s_dyn[];  // [kDownWarps][NT][4][32] warp partials, then [NT * 128] CTA partial
    auto s_part = reinterpret_cast<float (*)[NT][4][32]>(s_dyn);
    float *s_cta = s_dyn + kDownWarps * NT * 4 * 32;  // this CTA's partial tile, fragment order
    // the fused linear launched next may start once every CTA is past this
    // point (it reads x and W before waiting for t, so this grid releases it
    // only after its own predecessor has completed)
    pdl_wait_then_release();
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    // arrival counts of a split fused linear launched next (its predecessor,
    // which may still have used them, has completed)
    if (rank == 0)
        for (int i = threadIdx.x; i < ncounts; i += kDownWarps * 32) counts[i] = 0u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int64_t ra = g, rb = g + 8;
    const bool va = ra < M, vb = rb < M;
    const uint32_t *xa = reinterpret_cast<const uint32_t *>(x + (va ? ra : 0) * K);
    const uint32_t *xb = reinterpret_cast<const uint32_t *>(x + (vb ? rb : 0) * K);

    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;

    const int64_t ksteps = K / 16;
    constexpr int kAllWarps = kDownWarps * kDownCtas;
#pragma unroll 2
    for (int64_t kk = rank * kDownWarps + warp; kk < ksteps; kk += kAllWarps) {
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
    for (int o = threadIdx.x; o < NT * 4 * 32; o += kDownWarps * 32) {
        const int nt = o / 128, i = (o / 32) & 3, ln = o & 31;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < kDownWarps; ++w) v += s_part[w][nt][i][ln];
        s_cta[o] = v;
    }
    cluster.sync();  // every CTA's partial tile is complete and visible
    // 16 rows x kR columns = NT * 128 outputs; this CTA finishes a slice
    constexpr int kSlice = NT * 128 / kDownCtas;
    if (threadIdx.x < kSlice) {
        const int o = rank * kSlice + threadIdx.x;
        float v = 0.0f;
#pragma unroll
        for (int c = 0; c < kDownCtas; ++c) v += cluster.map_shared_rank(s_cta, c)[o];
        v *= s;
        const int nt = o / 128, i = (o / 32) & 3, ln = o & 31;
        const int row = (ln >> 2) + ((i & 2) ? 8 : 0);
        const int col = nt * 8 + 2 * (ln & 3) + (i & 1);
        if (row < M) {
            const __nv_bfloat16 hi = __float2bfloat16_rn(v);
            const __nv_bfloat16 lo = __float2bfloat16_rn(v - __bfloat162float(hi));
            t2[row * rp + col] = hi;
            t2[row * rp + kR + col] = lo;
        }
    }
    // zero padding columns [2r, rp)
    if (rank == 0) {
        for (int o = threadIdx.x; o < 16 * (rp - 2 * kR); o += kDownWarps * 32) {
            const int row = o / (rp - 2 * kR), col = 2 * kR + o % (rp - 2 * kR);
            if (row < M) t2[row * rp + col] = __float2bfloat16_rn(0.0f);
        }
    }
    cluster.sync();  // no CTA leaves while another may still read its partial tile
}

template <int kR>
cudaError_t launch_down(cudaStream_t stream, const __nv_bfloat16 *x, const __nv_bfloat16 *A, int64_t M, int64_t K,
                        float s, __nv_bfloat16 *t2, int rp, unsigned *counts, int ncounts) {
    const size_t smem = (size_t)(kDownWarps + 1) * (kR / 8) * 4 * 32 * sizeof(float);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_lora_down<kR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(k_lora_down<kR>, dim3(kDownCtas), dim3(kDownWarps * 32), smem, stream, kDownCtas, x, A, M, K,
                      s, t2, rp, counts, ncounts);
}

}  // namespace

int lora_rp(int r) { return ((2 * r + 63) / 64) * 64; }

// counts: ncounts arrival counts to zero for a split fused linear launched
// next (NULL, 0 when there is none).
cudaError_t launch_lora_down(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2,
                             unsigned *counts, int ncounts, cudaStream_t stream) {
    if (M > 16) return cudaErrorInvalidValue;  // larger M: launch_lora_down_tc
    const int rp = lora_rp(r);
    auto *xp = static_cast<const __nv_bfloat16 *>(x);
    auto *ap = static_cast<const __nv_bfloat16 *>(A);
    auto *tp = static_cast<__nv_bfloat16 *>(t2);
    cudaError_t e = cudaSuccess;
    switch (r) {
        case 16: e = launch_down<16>(stream, xp, ap, M, K, s, tp, rp, counts, ncounts); break;
        case 32: e = launch_down<32>(stream, xp, ap, M, K, s, tp, rp, counts, ncounts); break;
        case 64: e = launch_down<64>(stream, xp, ap, M, K, s, tp, rp, counts, ncounts); break;
        default: return cudaErrorInvalidValue;
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace nf4
