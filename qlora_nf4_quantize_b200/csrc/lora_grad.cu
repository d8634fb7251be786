// lora_grad.cu -- K9: the adapter gradients of the fused frozen-base LoRA
// linear ("QLoRA: Mathematical Foundations ...", section "Gradient
// Computation"), in the layout W[N, K], A[r, K], B[N, r], g = dL/dy [M, N]:
//   dA[j, k] = sum_m (s g B)[m, j] x[m, k]        fp32 [r, K]
//   dB[n, j] = sum_m g[m, n] (s x A^T)[m, j]      fp32 [N, r]
// Both are C[p, j] = sum_m X[m, p] T[m, j] with the contraction over the
// token rows of two row-major operands (X = x or g, T = s g B or s x A^T as
// computed by the down-projection kernels, a bf16 hi/lo pair [T_hi | T_lo]:
// both halves are multiplied and added, so T carries ~16 significant bits).
//
// Layout of the work: a CTA owns 128 columns p of X and one chunk of token
// rows; its 8 warps each own 16 p and all r columns j and run m16n8k16 MMAs
// whose A fragments (X^T) and B fragments (T) come from shared-memory tiles
// through ldmatrix.trans (the tiles stay in their row-major, token-major
// form).  Tiles of 32 token rows are double-buffered with cp.async.  Each
// chunk writes its fp32 partial; a second kernel adds the chunks in index
// order, so the result does not depend on timing.
#include "mbarrier.cuh"
#include "mma_util.cuh"

namespace nf4 {
namespace {

constexpr int kGP = 128;     // p columns per CTA
constexpr int kGMt = 32;     // token rows per staged tile
constexpr int kGThreadsG = 256;
constexpr int kGTargetCtas = 296;  // chunks chosen so that p-tiles x chunks ~ this (device independent)
constexpr int kXPitch = kGP * 2 + 16;  // bytes per staged X row (16-byte pad: conflict-free ldmatrix)

__device__ __forceinline__ void cp16(uint32_t dst, const void *src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t &a, uint32_t &b, uint32_t &c, uint32_t &d) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(a), "=r"(b), "=r"(c), "=r"(d)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x2_trans(uint32_t addr, uint32_t &a, uint32_t &b) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0, %1}, [%2];" : "=r"(a), "=r"(b) : "r"(addr));
}

// part[chunk][p][c] = sum over the chunk's token rows of X[m, p] T2[m, c],
// c < kC = 2 r (the hi and lo columns)
template <int kC>
__global__ void __launch_bounds__(kGThreadsG) k_lora_grad(const __nv_bfloat16 *__restrict__ X, int64_t P,
                                                          const __nv_bfloat16 *__restrict__ T, int64_t ldt,
                                                          int64_t M, int64_t m_chunk, float *__restrict__ part) {
    constexpr int NT = kC / 8;
    constexpr int kTPitch = kC * 2 + 16;  // bytes per staged T row
    __shared__ __align__(16) uint8_t sx[2][kGMt * kXPitch];
    __shared__ __align__(16) uint8_t st[2][kGMt * kTPitch];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t p0 = (int64_t)blockIdx.x * kGP;
    const int64_t mb = (int64_t)blockIdx.y * m_chunk;
    const int64_t me = mb + m_chunk < M ? mb + m_chunk : M;
    const int ntiles = me > mb ? (int)((me - mb + kGMt - 1) / kGMt) : 0;

    auto stage = [&](int tile, int buf) {
        const int64_t mt = mb + (int64_t)tile * kGMt;
        // X: 32 rows x 16 chunks of 16 bytes
        for (int c = threadIdx.x; c < kGMt * (kGP / 8); c += kGThreadsG) {
            const int row = c / (kGP / 8), ch = c % (kGP / 8);
            const int64_t m = mt + row, p = p0 + 8 * ch;
            const bool v = m < me && p < P;
            cp16(smem_addr(sx[buf] + row * kXPitch + ch * 16), v ? X + m * P + p : X, v);
        }
        // T2: 32 rows x kC / 8 chunks
        for (int c = threadIdx.x; c < kGMt * (kC / 8); c += kGThreadsG) {
            const int row = c / (kC / 8), ch = c % (kC / 8);
            const int64_t m = mt + row;
            const bool v = m < me;
            cp16(smem_addr(st[buf] + row * kTPitch + ch * 16), v ? T + m * ldt + 8 * ch : T, v);
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.0f;
    if (ntiles > 0) stage(0, 0);
    // ldmatrix row addresses: lane l feeds row (l % 8) of matrix (l / 8)
    const int mi = lane >> 3, ri = lane & 7;
    for (int t = 0; t < ntiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < ntiles) {
            stage(t + 1, buf ^ 1);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();
        const uint32_t xb = smem_addr(sx[buf]), tb = smem_addr(st[buf]);
#pragma unroll
        for (int ks = 0; ks < kGMt / 16; ++ks) {
            // A = X^T (16 p x 16 m): matrices (m 0-7, p 0-7), (m 0-7, p 8-15), (m 8-15, p 0-7), (m 8-15, p 8-15)
            uint32_t a[4];
            {
                const int m = 16 * ks + ri + 8 * (mi >> 1);
                const int pc = 16 * warp + 8 * (mi & 1);
                ldsm_x4_trans(xb + m * kXPitch + pc * 2, a[0], a[1], a[2], a[3]);
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                // B = T (16 m x 8 j): matrices (m 0-7, j), (m 8-15, j)
                uint32_t b0, b1;
                const int m = 16 * ks + ri + 8 * (mi & 1);
                ldsm_x2_trans(tb + m * kTPitch + (8 * nt) * 2, b0, b1);
                mma_bf16_16816(acc[nt], a, b0, b1);
            }
        }
        __syncthreads();  // the buffer is restaged two tiles later
    }
    // acc[nt]: rows p = 16 warp + g (+8), columns j = 8 nt + 2 tq (+1)
    const int g = lane >> 2, tq = lane & 3;
    float *out = part + (int64_t)blockIdx.y * P * kC;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t p = p0 + 16 * warp + g + 8 * (i >> 1);
            const int j = 8 * nt + 2 * tq + (i & 1);
            if (p < P) out[p * kC + j] = acc[nt][i];
        }
}

// out[p * sp + j * sj] = sum_c (part[c][p][j] + part[c][p][r + j]), c = 0, 1, ... in order
__global__ void k_grad_reduce(const float *__restrict__ part, int chunks, int64_t P, int r, float *__restrict__ out,
                              int64_t sp, int64_t sj) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= P * r) return;
    const int64_t p = i / r, j = i % r;
    const float *q = part + p * 2 * r + j;
    float v = 0.0f;
    for (int c = 0; c < chunks; ++c) v += q[(int64_t)c * P * 2 * r] + q[(int64_t)c * P * 2 * r + r];
    out[p * sp + j * sj] = v;
}

}  // namespace

// Token chunks of a gradient product over P columns (p-tiles x chunks ~ 296
// CTAs; independent of the device so that workspace sizes are too).
int64_t grad_chunks(int64_t M, int64_t P) {
    const int64_t ptiles = (P + kGP - 1) / kGP;
    int64_t c = (kGTargetCtas + ptiles - 1) / ptiles;
    const int64_t max_c = (M + kGMt - 1) / kGMt;
    if (c > max_c) c = max_c;
    return c < 1 ? 1 : c;
}

// out[p sp + j sj] = sum_m X[m, p] (T2[m, j] + T2[m, r + j]) in fp32 (part:
// grad_chunks(M, P) x P x 2r fp32 of scratch).
cudaError_t launch_lora_grad_product(const __nv_bfloat16 *X, int64_t P, const __nv_bfloat16 *T, int64_t ldt,
                                     int64_t M, int r, float *part, float *out, int64_t sp, int64_t sj,
                                     cudaStream_t stream) {
    const int64_t chunks = grad_chunks(M, P);
    const int64_t m_chunk = ((M + chunks - 1) / chunks + kGMt - 1) / kGMt * kGMt;
    const dim3 grid((unsigned)((P + kGP - 1) / kGP), (unsigned)chunks);
    switch (r) {
        case 16: k_lora_grad<32><<<grid, kGThreadsG, 0, stream>>>(X, P, T, ldt, M, m_chunk, part); break;
        case 32: k_lora_grad<64><<<grid, kGThreadsG, 0, stream>>>(X, P, T, ldt, M, m_chunk, part); break;
        case 64: k_lora_grad<128><<<grid, kGThreadsG, 0, stream>>>(X, P, T, ldt, M, m_chunk, part); break;
        default: return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t total = P * r;
    k_grad_reduce<<<(unsigned)((total + 255) / 256), 256, 0, stream>>>(part, (int)chunks, P, r, out, sp, sj);
    return cudaGetLastError();
}

}  // namespace nf4
