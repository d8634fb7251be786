// gemm_bwd.cu -- K8: the input gradient of the fused frozen-base LoRA linear
// on the tensor cores (tcgen05 / TMEM / TMA, sm_100a).
//
// "QLoRA: Mathematical Foundations ...", section "Gradient Computation": the
// activation gradient flows through both paths,
//   dx[m, k] = sum_n g[m, n] W~[n, k] + s sum_j u[m, j] A[j, k],  u = g B,
// in the layout W[N, K], A[r, K], B[N, r], g = dL/dy [M, N].  W~ is the bf16
// dequantized weight, bit-identical to nf4_dequantize's output; bf16 operands,
// fp32 accumulation, bf16 output.
//
// Unlike the forward, the contraction runs along W's rows (n), across the
// 64-blocks.  A CTA computes a 256 (tokens) x 256 (k) tile of dx as two MMA
// accumulators of 128 tokens each (512 tensor-memory columns):
//   D_h[m, k] += G[m, n] * W~[n, k],  M_mma = 128, N_mma = 256, K = 16
//   G  = g tile (256 tokens x 64 n) brought by TMA with 128-byte swizzle,
//        a K-major operand;
//   W~ = the dequantized weight tile (64 n x 256 k) written by the dequant
//        warpgroups into shared memory in its own row layout, as an MN-major
//        operand (instruction descriptor transpose bit): 128-byte swizzle
//        atoms of 8 rows n x 64 k, the four 64-k atoms of a row group 8 KB
//        apart (leading byte offset), row groups 1 KB apart (stride byte
//        offset).  A lane owns two rows (p and p + 32) of one 64-block,
//        dequantizes each with one register lookup table (mma_util.cuh) and
//        writes it with eight 16-byte stores; the 8 lanes of a store phase
//        write the 8 rows of one atom, so the stores are conflict-free;
// both operands come from shared memory (SS MMA).  Each dequantized weight
// feeds 256 tokens, as in the forward.  After the N / 64 weight steps, RP / 64
// extension steps add the LoRA term the same way: G' = [u_hi | u_lo | 0]
// (u scaled by s, as a bf16 hi/lo pair, from the down-projection kernel run
// on g with B^T) and W~' = rows of [A ; A ; 0] (A's own rows, no transpose).
//
// Warp roles (16 warps): warp 0 = TMA producer, warp 1 = TMEM allocator and
// MMA issuer (one elected thread), warps 4..15 = three dequant warpgroups
// (warpgroup h produces the k-steps with index % 3 == h) and, at the end, the
// epilogue (16 units of one accumulator and 32 columns spread over the
// warpgroups: tcgen05.ld, bf16, 64-byte row segments).  One full and one
// empty barrier per stage; every mbarrier wait is bounded as in the forward
// GEMM.
#include "mma_util.cuh"
#include "tc_util.cuh"

namespace nf4 {
namespace {

constexpr int kGM = 256;       // tokens per CTA (two accumulators of 128)
constexpr int kGN = 256;       // output columns k per CTA (MMA N)
constexpr int kGK = 64;        // contraction (n) per pipeline step
constexpr int kGStages = 3;
// dequant warpgroups: warpgroup h produces the k-steps with index % kGWG == h
#ifndef NF4_BWD_WG
#define NF4_BWD_WG 3
#endif
constexpr int kGWG = NF4_BWD_WG;
constexpr int kGThreads = 128 + 128 * kGWG;
constexpr uint32_t kGTmemCols = 512;
constexpr uint32_t kGStageBytes = kGM * kGK * 2;  // also the WT tile: kGN x kGK bf16
static_assert(kGM * kGK == kGN * kGK, "G and WT tiles have the same size");

// UMMA instruction descriptor, kind::f16: D fp32, A bf16 K-major, B bf16
// MN-major (bit 16), N = 256, M = 128.
constexpr uint32_t kGIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) | ((uint32_t)(kGN >> 3) << 17) |
                             ((uint32_t)(128 >> 4) << 24);
constexpr uint32_t kGAtomCol = kGK * 128;  // bytes of one 64-k column of atoms (64 rows x 128 B)

// MN-major operand in 128-byte swizzle atoms (8 rows along K x 64 elements
// along N): leading byte offset = distance between atoms along N, stride byte
// offset = distance between 8-row groups along K.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128_b(const void *p, uint32_t lbo_bytes) {
    const uint64_t addr = smem_addr(p);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// One lane of the (converged) warp, the same every time (the lowest).
__device__ __forceinline__ bool elect_one_lane() {
    uint32_t p;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(p));
    return p != 0;
}

struct __align__(1024) BwdSmem {
    uint8_t g[kGStages][kGStageBytes];
    uint8_t wt[kGStages][kGStageBytes];
    // full[s]: the g tile has landed (one arrival with its transaction bytes)
    // and the producing warpgroup has written the weight tile (one arrival
    // per warp); empty[s]: the MMAs that read stage s have completed (one
    // commit), awaited by the TMA producer and the dequant warpgroups alike
    uint64_t full[kGStages];
    uint64_t empty[kGStages];
    uint64_t acc_full;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

// 64 codes and the block constant of weight row n, k-block kb (whole block).
struct BlockCodes {
    uint32_t w[8];
    ScaleRaw sr;
};

template <int kMode>
__device__ __forceinline__ void load_block(const uint8_t *__restrict__ packed, const uint8_t *__restrict__ q8,
                                           const float *__restrict__ scales, int64_t n, int64_t K, int64_t kb,
                                           bool valid, BlockCodes &bc) {
    if (valid) {
        const uint4 *p = reinterpret_cast<const uint4 *>(packed + n * (K >> 1) + kb * 32);
        const uint4 u0 = __ldg(p), u1 = __ldg(p + 1);
        bc.w[0] = u0.x; bc.w[1] = u0.y; bc.w[2] = u0.z; bc.w[3] = u0.w;
        bc.w[4] = u1.x; bc.w[5] = u1.y; bc.w[6] = u1.z; bc.w[7] = u1.w;
        bc.sr = block_scale_load<kMode>(q8, scales, n * (K >> 6) + kb);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) bc.w[i] = 0x77777777u;  // code 7 = level 0
        bc.sr.q8 = 0;
        bc.sr.v = 0.0f;
    }
}

// byte offset of 16-byte chunk c (k = 8c .. 8c+7 of 64-k block a) of row n
// (0..63) in the MN-major swizzled weight tile
__device__ __forceinline__ uint32_t w_offset(int n, int a, int c) {
    return (uint32_t)a * kGAtomCol + (uint32_t)n * 128u + ((uint32_t)(c ^ (n & 7)) << 4);
}

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

template <int kMode>
__global__ void __launch_bounds__(kGThreads, 1)
    k_gemm_bwd(const __grid_constant__ CUtensorMap tmap_g, const __grid_constant__ CUtensorMap tmap_u, int64_t M,
               int64_t K, int64_t N, const uint8_t *__restrict__ packed, const uint8_t *__restrict__ q8,
               const float *__restrict__ scales, const float *__restrict__ offset,
               const __nv_bfloat16 *__restrict__ Al, int r, int rp, __nv_bfloat16 *__restrict__ dx, unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    BwdSmem &S = *reinterpret_cast<BwdSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int *abort = &S.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t k0 = (int64_t)blockIdx.x * kGN;
    const int64_t m0 = (int64_t)blockIdx.y * kGM;
    const int kn_steps = (int)((N + kGK - 1) / kGK);
    const int kt_total = kn_steps + (r > 0 ? rp / kGK : 0);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&S.full[s], 1 + 4);
            mbar_init(&S.empty[s], 1);
        }
        mbar_init(&S.acc_full, 1);
        mbar_init(&S.drain, 1);
        S.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&S.tmem_base)),
                     "r"(kGTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer: g tiles, then [u_hi | u_lo] tiles ----------------
        // (the whole warp runs the loop; one elected lane issues the copies)
        const bool leader = elect_one_lane();
        int issued = 0;
        for (int kt = 0; kt < kt_total; ++kt) {
            const int s = kt % kGStages;
            const uint32_t ph = (uint32_t)(kt / kGStages) & 1u;
            // u is written by the down-projection kernel launched just
            // before (programmatic dependent launch)
            if (kt == kn_steps) asm volatile("griddepcontrol.wait;" ::: "memory");
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&S.empty[s], ph ^ 1u, abort, err))) break;
            if (leader) {
                mbar_arrive_expect_tx(&S.full[s], kGStageBytes);
                if (kt < kn_steps) tma_load_2d(S.g[s], &tmap_g, &S.full[s], kt * kGK, (int)m0);
                else tma_load_2d(S.g[s], &tmap_u, &S.full[s], (kt - kn_steps) * kGK, (int)m0);
            }
            __syncwarp();
            issued = kt + 1;
        }
        if (leader) {
            for (int kt = issued - kGStages < 0 ? 0 : issued - kGStages; kt < issued; ++kt) {
                unsigned long long t0 = global_ns();
                while (!mbar_try_wait(&S.full[kt % kGStages], (uint32_t)(kt / kGStages) & 1u) &&
                       global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        // (the whole warp runs the loop; one elected lane issues the MMAs)
        const bool leader = elect_one_lane();
        {
            bool any = false;
            for (int kt = 0; kt < kt_total; ++kt) {
                const int s = kt % kGStages;
                const uint32_t ph = (uint32_t)(kt / kGStages) & 1u;
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(&S.full[s], ph, abort, err))) break;
                tc_fence_after();
                if (leader) {
                    const uint64_t a0 = smem_desc_sw128(S.g[s]);
                    const uint64_t a1 = smem_desc_sw128(S.g[s] + kGStageBytes / 2);  // tokens 128..255
                    const uint64_t bd = smem_desc_mn_sw128_b(S.wt[s], kGAtomCol);
#pragma unroll
                    for (int kk = 0; kk < kGK / 16; ++kk) {
                        const uint32_t acc = (kt | kk) != 0 ? 1u : 0u;
                        const uint64_t b = bd + (uint64_t)(kk * 2048 >> 4);  // 16 rows n = two atoms along K
                        tc_mma_ss(tmem, a0 + 2ull * kk, b, kGIdesc, acc);
                        tc_mma_ss(tmem + 256u, a1 + 2ull * kk, b, kGIdesc, acc);
                    }
                    tc_commit(&S.empty[s]);
                    if (kt == kt_total - 1) tc_commit(&S.acc_full);
                }
                __syncwarp();
                any = true;
            }
            if (leader && any && *abort) {  // drain our own MMAs before tensor memory is released
                tc_commit(&S.drain);
                unsigned long long t0 = global_ns();
                while (!mbar_try_wait(&S.drain, 0) && global_ns() - t0 < kWaitLimitNs) {
                }
            }
            __syncwarp();
        }
    } else if (warp >= 4) {
        // ---------------- dequant warpgroups (transposed tiles), then epilogue ----------------
        const int q = warp & 3;         // k-block of the tile / tensor-memory lane quarter
        const int h = (warp - 4) >> 2;  // warpgroup: k-steps with index % kGWG == h
        // rows p and p + 32 of the step: the 8 lanes a 16-byte store serves
        // together write 8 consecutive rows, whose swizzle phases differ
        const int p = lane;
        const int64_t kb = (k0 >> 6) + q;  // this lane's k-block of W
        const bool kvalid = kb * 64 < K;
        const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
        bool ok = true;
        BlockCodes ca, cb, na, nb;
        auto load_pair = [&](int kt, BlockCodes &x0, BlockCodes &x1) {
            const int64_t n = (int64_t)kt * kGK + p;
            load_block<kMode>(packed, q8, scales, n, K, kb, kvalid && n < N, x0);
            load_block<kMode>(packed, q8, scales, n + 32, K, kb, kvalid && n + 32 < N, x1);
        };
        if (h < kn_steps) load_pair(h, ca, cb);
        for (int kt = h; kt < kt_total; kt += kGWG) {
            const int s = kt % kGStages;
            const uint32_t ph = (uint32_t)(kt / kGStages) & 1u;
            const uint32_t tile = smem_addr(S.wt[s]);
            if (kt < kn_steps) {
                if (kt + kGWG < kn_steps) load_pair(kt + kGWG, na, nb);
                // word j of a row holds k = 2j (low half) and 2j + 1 (high half):
                // chunk c = words 4c .. 4c + 3; row p is dequantized before the
                // wait for the stage and stored after it, then row p + 32
                uint32_t v[32];
                {
                    const Lut la = make_lut(block_scale_finish<kMode>(ca.sr, mu));
#pragma unroll
                    for (int i = 0; i < 8; ++i) lut_lookup8(la, ca.w[i], v + 4 * i);
                }
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&S.empty[s], ph ^ 1u, abort, err));
                if (!ok) break;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    sts128(tile + w_offset(p, q, c), make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]));
                {
                    const Lut lb = make_lut(block_scale_finish<kMode>(cb.sr, mu));
#pragma unroll
                    for (int i = 0; i < 8; ++i) lut_lookup8(lb, cb.w[i], v + 4 * i);
                }
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    sts128(tile + w_offset(p + 32, q, c),
                           make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]));
                ca = na;
                cb = nb;
            } else {
                // rows j of [A ; A ; 0] (row j -> A[j mod r] for j < 2r), columns
                // k0 + 64 q .. + 63: rows p and p + 32 of the step
                const int e = kt - kn_steps;
                ok = __all_sync(0xFFFFFFFFu, mbar_wait(&S.empty[s], ph ^ 1u, abort, err));
                if (!ok) break;
                const int64_t k = k0 + 64 * q;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int j = 64 * e + p + 32 * i;
                    const bool v = j < 2 * r && k < K;
                    const uint4 *src = reinterpret_cast<const uint4 *>(Al + (int64_t)(v ? j % r : 0) * K + (v ? k : 0));
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        sts128(tile + w_offset(p + 32 * i, q, c), v ? __ldg(src + c) : make_uint4(0u, 0u, 0u, 0u));
                }
            }
            // the tile is read by the tensor cores (async proxy)
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.full[s]);
        }
        if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&S.acc_full, 0, abort, err));
        if (ok) {
            // Epilogue: 16 units (accumulator a of 128 tokens, 32-column chunk
            // c), unit a * 8 + c stored by warpgroup (a * 8 + c) % kGWG;
            // thread = token row.
            tc_fence_after();
#pragma unroll 1
            for (int u = h; u < 2 * (kGN / 32); u += kGWG) {
                const int a = u / (kGN / 32), c = u % (kGN / 32);
                const int64_t m = m0 + 128 * a + 32 * q + lane;
                const uint32_t base = tmem + ((uint32_t)(32 * q) << 16) + 256u * (uint32_t)a;
                uint32_t v[32];
                tc_load32(base + 32u * c, v);
                tc_wait_ld();
                const int64_t k = k0 + 32 * c;
                if (m < M && k < K) {
                    uint4 *dst = reinterpret_cast<uint4 *>(dx + m * K + k);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint32_t w[4];
#pragma unroll
                        for (int t = 0; t < 4; ++t)
                            w[t] = pack_bf16x2(__uint_as_float(v[8 * i + 2 * t]), __uint_as_float(v[8 * i + 2 * t + 1]));
                        dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kGTmemCols) : "memory");
    }
}

// dst[C, R] = src[R, C]^T for bf16 (32 x 32 tiles through shared memory)
__global__ void k_transpose_bf16(const __nv_bfloat16 *__restrict__ src, int64_t R, int64_t C,
                                 __nv_bfloat16 *__restrict__ dst) {
    __shared__ __nv_bfloat16 t[32][34];
    const int64_t r0 = (int64_t)blockIdx.y * 32, c0 = (int64_t)blockIdx.x * 32;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t rr = r0 + i, cc = c0 + threadIdx.x;
        if (rr < R && cc < C) t[i][threadIdx.x] = src[rr * C + cc];
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t cc = c0 + i, rr = r0 + threadIdx.x;
        if (rr < R && cc < C) dst[cc * R + rr] = t[threadIdx.x][i];
    }
}

template <int kMode>
cudaError_t launch_bwd_mode(const CUtensorMap &mg, const CUtensorMap &mu, int64_t M, int64_t K, int64_t N,
                            const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                            const __nv_bfloat16 *Al, int r, int rp, __nv_bfloat16 *dx, unsigned *err,
                            cudaStream_t stream) {
    const size_t smem = sizeof(BwdSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_gemm_bwd<kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((K + kGN - 1) / kGN), (unsigned)((M + kGM - 1) / kGM));
    cfg.blockDim = dim3(kGThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = r > 0 ? 1 : 0;  // overlap with the down-projection that precedes it
    return cudaLaunchKernelEx(&cfg, k_gemm_bwd<kMode>, mg, mu, M, K, N, packed, q8, scales, offset, Al, r, rp, dx,
                              err);
}

}  // namespace

cudaError_t launch_lora_down_tc(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2, int rp,
                                unsigned *err, cudaStream_t stream, int split, int max_ctas);
int lora_rp(int r);
int64_t grad_chunks(int64_t M, int64_t P);
cudaError_t launch_lora_grad_product(const __nv_bfloat16 *X, int64_t P, const __nv_bfloat16 *T, int64_t ldt,
                                     int64_t M, int r, float *part, float *out, int64_t sp, int64_t sj,
                                     cudaStream_t stream);
cudaError_t launch_lora_grad_product_tc(const __nv_bfloat16 *X, int64_t P, const __nv_bfloat16 *T2, int rp, int64_t M,
                                        int r, float *out, int64_t sp, int64_t sj, unsigned *err, cudaStream_t stream,
                                        int num_sms);

// dst[C, R] = src[R, C]^T (bf16)
cudaError_t launch_transpose_bf16(const __nv_bfloat16 *src, int64_t R, int64_t C, __nv_bfloat16 *dst,
                                  cudaStream_t stream) {
    const dim3 grid((unsigned)((C + 31) / 32), (unsigned)((R + 31) / 32));
    k_transpose_bf16<<<grid, dim3(32, 8), 0, stream>>>(src, R, C, dst);
    return cudaGetLastError();
}

static int64_t align256(int64_t b) { return (b + 255) & ~(int64_t)255; }

#ifndef NF4_GRAD_TC
#define NF4_GRAD_TC 1
#endif

namespace {

// Workspace of the backward pass (all 256-byte aligned):
//   u2 = [s g B hi | lo | 0]  bf16 [M, RP]   (dx extension and dA)
//   t2 = [s x A^T hi | lo | 0] bf16 [M, RP]  (dB)
//   B^T bf16 [r, N]
//   fp32 partials of dB (chunks x N x 2r) and of dA (chunks x K x 2r)
struct BwdWorkspace {
    int64_t u2, t2, bt, part_b, part_a, total;
};

BwdWorkspace bwd_layout(int64_t M, int64_t N, int64_t K, int r) {
    BwdWorkspace w{};
    if (r <= 0) return w;
    const int64_t rp = lora_rp(r);
    w.u2 = 0;
    w.t2 = w.u2 + align256(M * rp * 2);
    w.bt = w.t2 + align256(M * rp * 2);
    w.part_b = w.bt + align256((int64_t)r * N * 2);
    w.part_a = w.part_b + align256(grad_chunks(M, N) * N * 2 * r * 4);
    w.total = w.part_a + align256(grad_chunks(M, K) * K * 2 * r * 4);
    return w;
}

}  // namespace

int64_t lora_bwd_workspace_bytes(int64_t M, int64_t N, int64_t K, int r) { return bwd_layout(M, N, K, r).total; }

// The whole backward pass (see include/nf4.h, nf4_lora_linear_bwd).  Launch
// order: transposes, the down-projection(s), the dx GEMM (programmatic
// dependent launch on the last down-projection, whose result it reads only in
// its extension steps), then the two gradient products.
cudaError_t launch_lora_linear_bwd(const void *g, const void *x, int64_t M, int64_t K, int64_t N,
                                   const uint8_t *packed, const uint8_t *q8, const float *scales,
                                   const float *offset, const void *A, const void *B, int r, float s, void *dx,
                                   float *dA, float *dB, void *workspace, unsigned *err, cudaStream_t stream,
                                   int num_sms) {
    if (M > 0x7FFFFFFF || K > 0x7FFFFFFF || N > 0x7FFFFFFF) return cudaErrorInvalidValue;
    const int rp = r > 0 ? lora_rp(r) : 0;
    const BwdWorkspace L = bwd_layout(M, N, K, r);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    auto *u2 = reinterpret_cast<__nv_bfloat16 *>(ws + L.u2);
    auto *t2 = reinterpret_cast<__nv_bfloat16 *>(ws + L.t2);
    auto *Bt = reinterpret_cast<__nv_bfloat16 *>(ws + L.bt);
    const auto *Al = static_cast<const __nv_bfloat16 *>(A);
    const auto *gp = static_cast<const __nv_bfloat16 *>(g);
    const auto *xp = static_cast<const __nv_bfloat16 *>(x);
    cudaError_t e = cudaSuccess;
    // a long contraction over few 128-row tiles: split it over a 4-CTA cluster
    auto split_for = [&](int64_t kdim) { return ((M + 127) / 128) * 4 <= num_sms && kdim >= 2048 ? 4 : 0; };
    if (r > 0) {
        const bool need_u = dx != nullptr || dA != nullptr;
        if (need_u) {
            e = launch_transpose_bf16(static_cast<const __nv_bfloat16 *>(B), N, r, Bt, stream);
            if (e != cudaSuccess) return e;
        }
        if (need_u) {  // u2 = s g (B^T)^T = s g B
            e = launch_lora_down_tc(g, Bt, M, N, r, s, u2, rp, err, stream, split_for(N), 0);
            if (e != cudaSuccess) return e;
        }
        if (dB) {  // t2 = s x A^T
            e = launch_lora_down_tc(x, A, M, K, r, s, t2, rp, err, stream, split_for(K), 0);
            if (e != cudaSuccess) return e;
        }
    }
    if (dx) {
        CUtensorMap mg, mu;
        e = make_map(&mg, g, M, N, kGK, kGM, true);
        if (e != cudaSuccess) return e;
        e = r > 0 ? make_map(&mu, u2, M, rp, kGK, kGM, true) : make_map(&mu, g, M, N, kGK, kGM, true);
        if (e != cudaSuccess) return e;
        auto *dxp = static_cast<__nv_bfloat16 *>(dx);
        if (q8 == nullptr) e = launch_bwd_mode<2>(mg, mu, M, K, N, packed, q8, scales, offset, Al, r, rp, dxp, err, stream);
        else if (offset == nullptr)
            e = launch_bwd_mode<1>(mg, mu, M, K, N, packed, q8, scales, offset, Al, r, rp, dxp, err, stream);
        else e = launch_bwd_mode<0>(mg, mu, M, K, N, packed, q8, scales, offset, Al, r, rp, dxp, err, stream);
        if (e != cudaSuccess) return e;
    }
    // the adapter gradients: tensor-core products (NF4_GRAD_TC 0 selects the
    // warp-MMA form, which needs the fp32 partial scratch)
    if (dB) {
        e = NF4_GRAD_TC ? launch_lora_grad_product_tc(gp, N, t2, rp, M, r, dB, r, 1, err, stream, num_sms)
                        : launch_lora_grad_product(gp, N, t2, rp, M, r, reinterpret_cast<float *>(ws + L.part_b), dB,
                                                   r, 1, stream);
        if (e != cudaSuccess) return e;
    }
    if (dA) {
        e = NF4_GRAD_TC ? launch_lora_grad_product_tc(xp, K, u2, rp, M, r, dA, 1, K, err, stream, num_sms)
                        : launch_lora_grad_product(xp, K, u2, rp, M, r, reinterpret_cast<float *>(ws + L.part_a), dA,
                                                   1, K, stream);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace nf4
