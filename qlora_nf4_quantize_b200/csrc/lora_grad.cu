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
#include "mma_util.cuh"
#include "tc_util.cuh"

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

namespace {

// ---------------------------------------------------------------------------
// Tensor-core form (tcgen05): D[p, c] += X[m, p] T2[m, c] with M_mma = 128 p
// columns of X, N_mma = RP columns of T2 ([T_hi | T_lo | 0]), K = token rows.
// Both operands are read by TMA in their natural row-major form (boxes of 64
// columns x 64 token rows, 128-byte swizzle) and handed to the MMA as
// MN-major operands (instruction descriptor transpose bits): each 8-row x
// 128-byte swizzle atom holds 64 consecutive columns of 8 tokens; atoms along
// the columns are a box apart (leading byte offset 8 KB), atoms along the
// tokens 1 KB apart (stride byte offset).  One thread issues the TMA copies,
// another the MMAs (ring of kGStagesTc); a cluster of kSplit CTAs splits the token rows and
// adds its fp32 partials in rank order through distributed shared memory; the
// epilogue folds the hi and lo columns (c and c + r) and writes fp32.
constexpr int kGStagesTc = 5;
constexpr int kGBox = 64;                       // columns and token rows of one TMA box
constexpr uint32_t kGBoxBytes = kGBox * kGBox * 2;  // 8 KB

template <int kC>
struct __align__(1024) GradSmem {
    uint8_t a[kGStagesTc][2][kGBoxBytes];         // X: p 0-63, p 64-127
    uint8_t b[kGStagesTc][kC / kGBox][kGBoxBytes];  // T2: c in boxes of 64
    uint64_t full[kGStagesTc];
    uint64_t empty[kGStagesTc];
    uint64_t acc_full;
    uint32_t tmem_base;
    int abort;
};

// MN-major operand in 128-byte swizzle atoms (8 rows along K x 64 elements
// along M or N): leading byte offset = distance between atoms along M/N,
// stride byte offset = distance between 8-row groups along K.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(const void *p, uint32_t lbo_bytes) {
    const uint64_t addr = smem_addr(p);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;                      // start address
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;  // leading byte offset: next 64-column atom
    d |= (uint64_t)(1024 >> 4) << 32;                   // stride byte offset: next 8 token rows
    d |= (uint64_t)1 << 46;                             // descriptor version for tcgen05
    d |= (uint64_t)2 << 61;                             // SWIZZLE_128B
    return d;
}

__device__ __forceinline__ void cluster_sync_all_g() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int kR, int kSplit>
__global__ void __launch_bounds__(128, 1)
    k_grad_tc(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_t, int64_t M,
              int64_t P, float *__restrict__ out, int64_t sp, int64_t sj, unsigned *err) {
    constexpr int kC = (2 * kR + 63) / 64 * 64;  // RP: columns of [T_hi | T_lo | 0]
    constexpr int r = kR;
    // D fp32, A bf16, B bf16, A and B MN-major (bits 15, 16), N = kC, M = 128
    constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                                ((uint32_t)(kC >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
    constexpr uint32_t kStageBytes = (2 + kC / kGBox) * kGBoxBytes;
    extern __shared__ uint8_t smem_raw[];
    GradSmem<kC> &S =
        *reinterpret_cast<GradSmem<kC> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int *abort = &S.abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    uint32_t rank;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
    const int64_t p0 = (int64_t)blockIdx.y * 128;
    const int kt_all = (int)((M + kGBox - 1) / kGBox);
    const int kt_begin = (int)((int64_t)rank * kt_all / kSplit);
    const int kt_total = (int)((int64_t)(rank + 1) * kt_all / kSplit) - kt_begin;
    if (threadIdx.x == 0) {
        for (int st = 0; st < kGStagesTc; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], 1);
        }
        mbar_init(&S.acc_full, 1);
        S.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&S.tmem_base)),
                     "r"((uint32_t)kC)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (threadIdx.x == 0 && kt_total > 0) {
        // producer: the X and T2 boxes of every 64-token step, kGStagesTc ahead
        int issued = 0;
        for (; issued < kt_total; ++issued) {
            const int st = issued % kGStagesTc;
            const uint32_t ph = (uint32_t)(issued / kGStagesTc) & 1u;
            if (!mbar_wait(&S.empty[st], ph ^ 1u, abort, err)) break;
            mbar_arrive_expect_tx(&S.full[st], kStageBytes);
            const int m = (kt_begin + issued) * kGBox;
            tma_load_2d(S.a[st][0], &tmap_x, &S.full[st], (int)p0, m);
            tma_load_2d(S.a[st][1], &tmap_x, &S.full[st], (int)p0 + kGBox, m);
#pragma unroll
            for (int i = 0; i < kC / kGBox; ++i) tma_load_2d(S.b[st][i], &tmap_t, &S.full[st], kGBox * i, m);
        }
        if (*abort) {  // every issued load lands before the CTA may exit
            for (int kt = issued - kGStagesTc < 0 ? 0 : issued - kGStagesTc; kt < issued; ++kt) {
                unsigned long long t0 = global_ns();
                while (!mbar_try_wait(&S.full[kt % kGStagesTc], (uint32_t)(kt / kGStagesTc) & 1u) &&
                       global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else if (threadIdx.x == 32 && kt_total > 0) {
        // MMA issuer, its own thread so that copies and MMAs overlap
        for (int kt = 0; kt < kt_total; ++kt) {
            const int st = kt % kGStagesTc;
            if (!mbar_wait(&S.full[st], (uint32_t)(kt / kGStagesTc) & 1u, abort, err)) break;
            tc_fence_after();
            const uint64_t ad = smem_desc_mn_sw128(S.a[st][0], kGBoxBytes);
            const uint64_t bd = smem_desc_mn_sw128(S.b[st][0], kGBoxBytes);
#pragma unroll
            for (int kk = 0; kk < kGBox / 16; ++kk)  // 16 token rows = two 8-row atoms
                tc_mma_ss(tmem, ad + (uint64_t)(kk * 2048 >> 4), bd + (uint64_t)(kk * 2048 >> 4), kIdesc,
                          (kt | kk) != 0 ? 1u : 0u);
            tc_commit(&S.empty[st]);
        }
        tc_commit(&S.acc_full);
    }
    __syncwarp();
    // fold hi + lo into this CTA's partial tile, column-major [r][128] fp32, in
    // the idle operand ring (every MMA that read it has completed)
    float *part = reinterpret_cast<float *>(&S.a[0][0][0]);
    const int row = 32 * warp + lane;
    if (kt_total > 0 && __all_sync(0xFFFFFFFFu, mbar_wait(&S.acc_full, 0, abort, err))) {
        tc_fence_after();
        const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
        for (int j0 = 0; j0 < r; j0 += 16) {
            uint32_t hi[32], lo[32];
            tc_load32(taddr + (uint32_t)(j0 & ~31), hi);
            tc_load32(taddr + (uint32_t)((r + j0) & ~31), lo);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j)
                part[(j0 + j) * 128 + row] =
                    __uint_as_float(hi[(j0 & 31) + j]) + __uint_as_float(lo[((r + j0) & 31) + j]);
        }
    } else {
        for (int j = 0; j < r; ++j) part[j * 128 + row] = 0.0f;
    }
    if constexpr (kSplit > 1) cluster_sync_all_g();
    {
        // CTA `rank` finishes rows [128 rank / kSplit, 128 (rank + 1) / kSplit):
        // thread t takes row (t % rows) and every (128 / rows)-th column
        constexpr int kRows = 128 / kSplit;
        const int t = threadIdx.x;
        const int rl = kRows * (int)rank + t % kRows;
        const int64_t p = p0 + rl;
        for (int j = t / kRows; j < r; j += 128 / kRows) {
            float v = 0.0f;
#pragma unroll
            for (int c = 0; c < kSplit; ++c) {
                uint32_t addr;
                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                             : "=r"(addr)
                             : "r"(smem_addr(part + j * 128 + rl)), "r"((uint32_t)c));
                float x;
                asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(x) : "r"(addr) : "memory");
                v += x;
            }
            if (p < P) out[p * sp + j * sj] = v;
        }
    }
    if constexpr (kSplit > 1) cluster_sync_all_g();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"((uint32_t)kC)
                     : "memory");
    }
}

template <int kR, int kSplit>
cudaError_t launch_grad_tc_k(const CUtensorMap &mx, const CUtensorMap &mt, int64_t M, int64_t P, float *out,
                             int64_t sp, int64_t sj, unsigned *err, cudaStream_t stream) {
    constexpr int kC = (2 * kR + 63) / 64 * 64;
    const size_t smem = sizeof(GradSmem<kC>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_grad_tc<kR, kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kSplit, (unsigned)((P + 127) / 128));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kSplit;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_grad_tc<kR, kSplit>, mx, mt, M, P, out, sp, sj, err);
}

template <int kR>
cudaError_t launch_grad_tc_r(const CUtensorMap &mx, const CUtensorMap &mt, int64_t M, int64_t P, float *out,
                             int64_t sp, int64_t sj, unsigned *err, cudaStream_t stream, int split) {
    if (split >= 4) return launch_grad_tc_k<kR, 4>(mx, mt, M, P, out, sp, sj, err, stream);
    if (split == 2) return launch_grad_tc_k<kR, 2>(mx, mt, M, P, out, sp, sj, err, stream);
    return launch_grad_tc_k<kR, 1>(mx, mt, M, P, out, sp, sj, err, stream);
}

}  // namespace

// Tensor-core gradient product: out[p sp + j sj] = sum_m X[m, p] (T2[m, j] +
// T2[m, r + j]); X bf16 [M, P] (P % 8 == 0), T2 bf16 [M, RP].
cudaError_t launch_lora_grad_product_tc(const __nv_bfloat16 *X, int64_t P, const __nv_bfloat16 *T2, int rp, int64_t M,
                                        int r, float *out, int64_t sp, int64_t sj, unsigned *err, cudaStream_t stream,
                                        int num_sms) {
    CUtensorMap mx, mt;
    cudaError_t e = make_map(&mx, X, M, P, kGBox, kGBox, true);
    if (e != cudaSuccess) return e;
    e = make_map(&mt, T2, M, rp, kGBox, kGBox, true);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (P + 127) / 128;
    const int split = tiles * 4 <= num_sms ? 4 : (tiles * 2 <= num_sms ? 2 : 1);
    switch (r) {
        case 16: return launch_grad_tc_r<16>(mx, mt, M, P, out, sp, sj, err, stream, split);
        case 32: return launch_grad_tc_r<32>(mx, mt, M, P, out, sp, sj, err, stream, split);
        case 64: return launch_grad_tc_r<64>(mx, mt, M, P, out, sp, sj, err, stream, split);
        default: return cudaErrorInvalidValue;
    }
}

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
