// gemm_tc.cu -- K5: fused NF4-dequantizing tensor-core GEMM for large token
// counts (tcgen05 / TMEM / TMA, sm_100a).
//
//   y[M, N] = x[M, K] W~[N, K]^T + [t_hi | t_lo | 0][M, RP] [B | B | 0][N, RP]^T
//
// "QLoRA: Mathematical Foundations ...", section "Forward Pass Computation":
// the NF4 weight is dequantized on the fly into on-chip tiles and never
// written to global memory; bf16 operands, fp32 accumulation, bf16 output.
// W~ is bit-identical to the bf16 output of nf4_dequantize.
//
// One CTA computes a 128 (weight rows) x 256 (tokens) tile of y^T:
//   MMA  D[n, m] += A[n, k] * X[m, k],   M_mma = 128, N_mma = 256, K = 16
//   A = W~ (bf16) lives in tensor memory: three dequant warpgroups turn the
//       packed nibbles of a 64-wide k-step into bf16 in registers (one scale
//       and one register lookup table per 64-block per thread, see
//       mma_util.cuh) and store them with tcgen05.st; no shared memory is
//       used for the weight.
//   X = x tile (256 tokens x 64 k, bf16) brought in by TMA with 128-byte
//       swizzle into a 6-stage shared-memory ring.
//   D = fp32 accumulators in tensor memory (256 columns).
// After the K/64 weight steps the same pipeline runs RP/64 extension steps in
// which the warpgroups copy rows of [B | B | 0] into tensor memory and TMA
// brings tiles of the [t_hi | t_lo | 0] workspace: the LoRA term is summed by
// the same MMAs into the same accumulators.
//
// Warp roles (16 warps): warp 0 = TMA producer, warp 1 = TMEM allocator and
// MMA issuer (one elected lane of the converged warp), warps 4..15 = three
// dequant warpgroups (warpgroup h produces the k-steps with index = h mod 3)
// and, at the end, the epilogue (tcgen05.ld, bf16 conversion, one TMA store
// of y).  The same pipeline with a 16-token tile can serve decode calls of 9
// to 16 tokens, split over the SMs (stream-K, see TmemPlan below): in a
// library built with NF4_SMALL_M_TC_FROM=9 (linear.cu); by default the
// decode kernel (decode.cu) takes every call of up to 16 tokens.
//
// Every mbarrier wait is bounded (about one second of %globaltimer): on
// expiry the waiter raises a CTA-wide abort flag and the device error word,
// every role leaves its loop, the MMA issuer drains its own MMAs, the TMA
// producer drains its own loads, and tensor memory is released before the
// CTA exits.  nf4_device_status() reports the expiry as NF4_ERR_TIMEOUT.
#include "mma_util.cuh"
#include "streamk.h"
#include "tc_util.cuh"

namespace nf4 {
namespace {

constexpr int kBN = 128;                   // weight rows per CTA (MMA M)
constexpr int kBK = 64;                    // k per pipeline step
#ifndef NF4_GEMM_STAGES
#define NF4_GEMM_STAGES 6
#endif
#ifndef NF4_GEMM_SUB
#define NF4_GEMM_SUB 1
#endif
// Dequant warpgroups: warpgroup h produces the k-steps with index % WG == h.
#ifndef NF4_GEMM_WG
#define NF4_GEMM_WG 3
#endif
// Dequantization lookup per warpgroup: bit h set = warpgroup h uses the
// shared-memory pair table (one shared load per two weights), clear = the
// register lookup table (byte permutes on the integer pipe).  Mixing the two
// spreads the work over the integer pipe and the shared-memory pipe.
#ifndef NF4_GEMM_LUT_MASK
#define NF4_GEMM_LUT_MASK 0
#endif
constexpr int kLutMask = NF4_GEMM_LUT_MASK;
// k-steps of packed codes each dequant thread keeps in flight
#ifndef NF4_GEMM_PF
#define NF4_GEMM_PF 1
#endif

constexpr uint32_t pow2_at_least(uint32_t v) {
    uint32_t p = 32;
    while (p < v) p <<= 1;
    return p;
}

// Token tile BT (MMA N), pipeline depth and dequant warpgroups of one
// instantiation: BT = 256 for the large-M GEMM; BT = 16 serves 9 to 16 tokens
// (a rate bound by the dequantization, the same for any token count up to 16;
// below 9 tokens the warp-MMA GEMV kernels are faster), normally split over
// the SMs.
constexpr uint32_t AccColsFor(int bt) { return bt < 32 ? 32u : (uint32_t)bt; }

template <int BT_, int STAGES_, int WG_, int SUB_, bool PAIR_ = false>
struct TileCfg {
    static constexpr int BT = BT_, Stages = STAGES_, WG = WG_;
    // CTA pair (cta_group::2): the two CTAs of a 2-CTA cluster own weight
    // tiles 2p and 2p + 1 and the same token tile; the even CTA issues MMAs
    // of M = 256 (its 128 rows and its partner's, each in its own tensor
    // memory) against the whole token tile, of which each CTA loads half.
    static constexpr bool Pair = PAIR_;
    static constexpr int XRows = PAIR_ ? BT_ / 2 : BT_;  // tokens of the x tile this CTA loads
    // k-steps of 64 per pipeline stage: the stage's barriers, its TMA
    // transaction and its MMA issue are shared by SUB k-steps
    static constexpr int Sub = SUB_;
    static constexpr int Threads = 128 + 128 * WG;
    // two CTAs per SM when both fit (registers at 128 per thread, tensor
    // memory at 256 columns each)
    static constexpr int MinBlocks =
        (!PAIR_ && Threads <= 256 && AccColsFor(BT_) + 32 * SUB_ * STAGES_ <= 256) ? 2 : 1;
    static constexpr uint32_t AccCols = AccColsFor(BT);     // accumulator: columns [0, AccCols)
    // A of k-step j of stage s: columns [ACol + 32 (Sub s + j), +32)
    static constexpr uint32_t ACol = AccCols;
    static constexpr uint32_t TmemCols = pow2_at_least(AccCols + 32 * Sub * Stages);
    static constexpr uint32_t XSubBytes = XRows * kBK * 2;  // one 64-wide k-step of (this CTA's part of) x
    static constexpr uint32_t XStageBytes = Sub * XSubBytes;
    // UMMA instruction descriptor, kind::f16: D fp32, A bf16, B bf16, both
    // K-major, N = BT, M = 128 (256 for a pair).
    static constexpr uint32_t Idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BT >> 3) << 17) |
                                      ((uint32_t)((PAIR_ ? 2 * kBN : kBN) >> 4) << 24);
    static_assert(TmemCols <= 512, "tensor memory: accumulator + 32 columns per A stage");
    static_assert(BT % 16 == 0 && BT >= 16 && BT <= 256, "MMA N for M = 128");
};

#ifndef NF4_GEMM_BT
#define NF4_GEMM_BT 256
#endif
using CfgLarge = TileCfg<NF4_GEMM_BT, NF4_GEMM_STAGES, NF4_GEMM_WG, NF4_GEMM_SUB>;
// Large-M calls on CTA pairs (cta_group::2) instead of single CTAs.  Exact
// (every linear parity test passes with it) but not the default: on B200 the
// training shape took 573.5 us against 430.6 us for single CTAs (six
// stages): the pair halves the MMA instructions and each CTA's share of the
// token tile, but every stage then waits for the slower of two SMs' dequant
// warps and for the remote arrivals, while each SM still dequantizes a whole
// 128-row tile per token tile.
#ifndef NF4_GEMM_PAIR
#define NF4_GEMM_PAIR 0
#endif
#ifndef NF4_GEMM_PAIR_STAGES
#define NF4_GEMM_PAIR_STAGES 6
#endif
using CfgPair = TileCfg<256, NF4_GEMM_PAIR_STAGES, 3, 1, true>;
static_assert(CfgPair::Stages * CfgPair::XStageBytes >= 256 * 128 * 2, "the y staging tile fits in the x ring");
#ifndef NF4_GEMV_TC_WG
#define NF4_GEMV_TC_WG 3
#endif
#ifndef NF4_GEMV_TC_STAGES
#define NF4_GEMV_TC_STAGES 6
#endif
#ifndef NF4_GEMV_TC_SUB
#define NF4_GEMV_TC_SUB 1
#endif
using CfgSmall = TileCfg<16, NF4_GEMV_TC_STAGES, NF4_GEMV_TC_WG, NF4_GEMV_TC_SUB>;

template <class C>
struct __align__(1024) SmemLayout {
    uint8_t x[C::Stages][C::XStageBytes];
    // full[s]: the x tile has landed (one arrival with its transaction
    // bytes) and the dequant warpgroup has stored the weight tile (128
    // arrivals); empty[s]: the MMAs that read stage s have completed (one
    // commit), awaited by the TMA producer and the dequant warpgroups alike
    uint64_t full[C::Stages];
    uint64_t empty[C::Stages];
    float2 pairs[kLutMask != 0 ? kPairTableFloat2 : 1];
    uint64_t acc_full;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int last[2];  // stream-K: this CTA adds up tile tile0 + h (h = segment)
};

__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// The same MMA for a CTA pair (issued by the even CTA): A from both CTAs'
// tensor memory (same address), B from both CTAs' shared memory (same
// offset, each holding half of the N rows), D in both CTAs' tensor memory.
__device__ __forceinline__ void tc_mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// One lane of the (converged) warp, the same every time: elect.sync picks
// the lowest active lane.
__device__ __forceinline__ bool elect_one() {
    uint32_t p;
    asm volatile(
        "{\n\t.reg .pred P;\n\t"
        "elect.sync _|P, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(p));
    return p != 0;
}

// The packed codes (8 words) and block constant of one 64-wide k-step of
// weight row n; all-zero-code words outside the matrix.
struct StepCodes {
    uint32_t w[8];
    ScaleRaw sr;  // block constant operands (decoded at use)
};

template <int kMode>
__device__ __forceinline__ void load_step(const uint8_t *__restrict__ packed, const uint8_t *__restrict__ q8,
                                          const float *__restrict__ scales, float /*mu*/, int64_t n, int64_t K,
                                          int64_t kt, bool valid, StepCodes &sc) {
    if (valid) {
        const uint4 *p = reinterpret_cast<const uint4 *>(packed + n * (K >> 1) + kt * 32);
        const uint4 u0 = __ldg(p), u1 = __ldg(p + 1);
        sc.w[0] = u0.x; sc.w[1] = u0.y; sc.w[2] = u0.z; sc.w[3] = u0.w;
        sc.w[4] = u1.x; sc.w[5] = u1.y; sc.w[6] = u1.z; sc.w[7] = u1.w;
        sc.sr = block_scale_load<kMode>(q8, scales, n * (K >> 6) + kt);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) sc.w[i] = 0x77777777u;
        sc.sr.q8 = 0;
        sc.sr.v = 0.0f;
    }
}

// 64 bf16 weights (one k-step) as 32 bf16x2 words, word j = (element 2j low
// half, element 2j+1 high half).
template <int kMode>
__device__ __forceinline__ void dequant_step(const StepCodes &sc, float mu, uint32_t out[32]) {
    const Lut lut = make_lut(block_scale_finish<kMode>(sc.sr, mu));
#pragma unroll
    for (int i = 0; i < 8; ++i) lut_lookup8(lut, sc.w[i], out + 4 * i);
}

template <int kMode>
__device__ __forceinline__ void dequant_step_smem(const StepCodes &sc, float mu, const float2 *tbl_lane,
                                                  uint32_t out[32]) {
    const float c = block_scale_finish<kMode>(sc.sr, mu);
#pragma unroll
    for (int s = 0; s < 16; ++s) pair_lookup4(tbl_lane, sc.w[s >> 1] >> ((s & 1) * 16), c, out[2 * s], out[2 * s + 1]);
}

// 64 columns [64 e, 64 e + 64) of the row n of [B | B | 0] (bf16 pairs):
// column j is B[n, j mod r] for j < 2r, else 0.  The row is read with
// 16-byte loads (rows of 2r bytes, 16-byte aligned: r = 16, 32, 64); since 64 is a
// multiple of r, column 64 e + 2c takes word c mod (r / 2) of the row.
template <int R>
__device__ __forceinline__ void lora_step_r(const __nv_bfloat16 *__restrict__ Bl, int64_t n, bool valid, int e,
                                            uint32_t out[32]) {
    // the row's R / 2 words go straight into out[0 .. R/2); the rest repeat
    // them ([B | B]) or are zero (columns >= 2r)
    const uint4 *src = reinterpret_cast<const uint4 *>(Bl + (valid ? n : 0) * R);
#pragma unroll
    for (int i = 0; i < R / 8; ++i) {
        const uint4 u = valid ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
        out[4 * i] = u.x; out[4 * i + 1] = u.y; out[4 * i + 2] = u.z; out[4 * i + 3] = u.w;
    }
#pragma unroll
    for (int c = R / 2; c < 32; ++c) out[c] = (64 * e + 2 * c < 2 * R) ? out[c % (R / 2)] : 0u;
}

__device__ __forceinline__ void lora_step(const __nv_bfloat16 *__restrict__ Bl, int r, int64_t n, bool valid,
                                          int e, uint32_t out[32]) {
    if (r == 16) lora_step_r<16>(Bl, n, valid, e, out);
    else if (r == 32) lora_step_r<32>(Bl, n, valid, e, out);
    else lora_step_r<64>(Bl, n, valid, e, out);
}

// Stream-K split (kSK, 16-token tile only).  The CTAs share out the
// sequence of (weight tile, k-step) pairs, tile after tile, in equal
// contiguous ranges [c T / G, (c + 1) T / G) of the T = tiles x kt_total
// steps, so that every SM streams the same share of the weight whatever the
// number of 128-row tiles.  With at least as many CTAs as tiles a range
// covers the end of one tile and the start of the next at most; each part
// (segment) accumulates into its own tensor-memory columns and is written as
// an fp32 partial tile [16 tokens][128 rows].  The CTA that completes a
// tile's arrival count adds the tile's partials in CTA order (so the result
// does not depend on timing) and writes y.  The counts are zeroed by the
// kernel launched just before (programmatic dependent launch), which is
// awaited before the first count.
template <class C, bool kSK>
struct TmemPlan {
    static constexpr int kAccs = kSK ? 2 : 1;                   // accumulators (segments)
    static constexpr uint32_t ACol = kAccs * C::AccCols;        // first A column
    static constexpr uint32_t Cols = pow2_at_least(ACol + 32 * C::Sub * C::Stages);
    static_assert(Cols <= 512, "tensor memory: accumulators + 32 columns per A stage");
    static_assert(!kSK || C::BT == 16, "stream-K split: 16-token tile");
    static_assert(!kSK || C::WG >= 2, "stream-K split: one epilogue warpgroup per segment");
};

// Partial tile of one segment: [16 tokens][128 rows] fp32.
constexpr int kPartialFloats = 16 * 128;
// Most CTAs of a split launch (the partials are sized for them) and fewest
// k-steps per CTA worth a split.
constexpr int kStreamKMaxCtas = 192;
constexpr int kStreamKMinSteps = 8;


template <int kMode, class C, bool kSK>
__global__ void __launch_bounds__(C::Threads, C::MinBlocks)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_t,
              const __grid_constant__ CUtensorMap tmap_y, int64_t M,
              int64_t K, int64_t N, const uint8_t *__restrict__ packed, const uint8_t *__restrict__ q8,
              const float *__restrict__ scales, const float *__restrict__ offset,
              const __nv_bfloat16 *__restrict__ Bl, int r, int rp, __nv_bfloat16 *__restrict__ y,
              float *__restrict__ partials, unsigned *__restrict__ counts, unsigned *err) {
    extern __shared__ uint8_t smem_raw[];
    constexpr int kBT = C::BT, kStages = C::Stages, kWG = C::WG, kSub = C::Sub;
    constexpr bool kPair = C::Pair;
    static_assert(!(kPair && kSK), "a CTA pair runs whole tiles");
    constexpr uint32_t kTmemCols = TmemPlan<C, kSK>::Cols, kAccCol = 0, kACol = TmemPlan<C, kSK>::ACol,
                       kXSubBytes = C::XSubBytes, kXStageBytes = C::XStageBytes;
    SmemLayout<C> &S =
        *reinterpret_cast<SmemLayout<C> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int *abort = &S.abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m0 = (int64_t)blockIdx.y * kBT;
    const int kw_steps = (int)(K / kBK);
    const int kt_total = kw_steps + (r > 0 ? rp / kBK : 0);
    // This CTA's k-steps: i = 0 .. steps-1 run over weight tile tile0 from
    // k-step kt_first, and from i = i_next over tile tile0 + 1 from k-step 0
    // (stream-K only; otherwise one whole tile, i_next = steps).
    int64_t tile0 = blockIdx.x, total = 0;
    int kt_first = 0, steps = kt_total, i_next = kt_total;
    if constexpr (kSK) {
        total = ((N + kBN - 1) / kBN) * kt_total;
        const int64_t lo = nf4_sk_begin(blockIdx.x, total, gridDim.x);
        const int64_t hi = nf4_sk_begin(blockIdx.x + 1, total, gridDim.x);
        tile0 = lo / kt_total;
        kt_first = (int)(lo - tile0 * kt_total);
        steps = (int)(hi - lo);
        i_next = kt_total - kt_first;
    }
    const int64_t n0 = tile0 * kBN;
    // segment (0 or 1) and k-step of step i
    auto seg_of = [&](int i) { return kSK ? (i >= i_next ? 1 : 0) : 0; };
    auto kt_of = [&](int i) { return kSK ? (i >= i_next ? i - i_next : kt_first + i) : i; };
    const int kg_total = (steps + kSub - 1) / kSub;  // pipeline stages (groups of kSub k-steps)
    // Programmatic dependent launch.  With an adapter the grid before this one
    // is the down-projection, which releases it only after its own
    // predecessor completed: x and W may be read at once, t only after the
    // wait in the extension steps.  The split launch is always preceded by a
    // kernel of that kind (the down-projection, or the zeroing of its arrival
    // counts).  Otherwise, without an adapter, wait before reading anything.
    if (!kSK && r <= 0) asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    // CTA pair: rank 0 issues the MMAs and owns the full barriers, which
    // count its own and its partner's dequant arrivals
    const uint32_t rank = kPair ? cluster_ctarank() : 0u;
    const bool issuer = rank == 0;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&S.full[s], 1 + 128 * (kPair ? 2 : 1));
            mbar_init(&S.empty[s], 1);
        }
        mbar_init(&S.acc_full, 1);
        mbar_init(&S.drain, 1);
        S.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if constexpr (kLutMask != 0) fill_pair_table(S.pairs);
    if (warp == 1) {
        if constexpr (kPair) {  // the same warp of both CTAs: one address, valid in both
            asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_addr(&S.tmem_base)),
                         "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
        } else {
            asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                             smem_addr(&S.tmem_base)),
                         "r"(kTmemCols)
                         : "memory");
            asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    // a pair: both CTAs' barriers are initialised before either signals the other's
    if constexpr (kPair) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        // (the whole warp runs the loop; one elected lane issues the copies)
        const bool leader = elect_one();
        int issued = 0;
        bool t_ready = false;
        for (int g = 0; g < kg_total; ++g) {
            const int s = g % kStages;
            const uint32_t ph = (uint32_t)(g / kStages) & 1u;
            const int i0 = g * kSub;
            const int nsub = steps - i0 < kSub ? steps - i0 : kSub;
            // the t workspace is written by the down-projection kernel
            // launched just before (programmatic dependent launch): wait
            // before the first extension step
            if (!t_ready && kt_of(i0 + nsub - 1) >= kw_steps) {
                asm volatile("griddepcontrol.wait;" ::: "memory");
                t_ready = true;
            }
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&S.empty[s], ph ^ 1u, abort, err))) break;
            if (leader) {
                if constexpr (kPair) {
                    // each CTA loads its half of the token tile; the bytes of
                    // both halves are counted on the even CTA's full barrier
                    if (issuer) mbar_arrive_expect_tx(&S.full[s], 2u * (uint32_t)nsub * kXSubBytes);
                    const uint32_t bar = cluster_addr(&S.full[s], 0);
                    const int row = (int)m0 + (int)rank * C::XRows;
                    for (int j = 0; j < nsub; ++j) {
                        const int kt = kt_of(i0 + j);
                        uint8_t *dst = S.x[s] + j * kXSubBytes;
                        if (kt < kw_steps) tma_load_2d_pair(dst, &tmap_x, bar, kt * kBK, row);
                        else tma_load_2d_pair(dst, &tmap_t, bar, (kt - kw_steps) * kBK, row);
                    }
                } else {
                    mbar_arrive_expect_tx(&S.full[s], (uint32_t)nsub * kXSubBytes);
                    for (int j = 0; j < nsub; ++j) {
                        const int kt = kt_of(i0 + j);
                        uint8_t *dst = S.x[s] + j * kXSubBytes;
                        if (kt < kw_steps) tma_load_2d(dst, &tmap_x, &S.full[s], kt * kBK, (int)m0);
                        else tma_load_2d(dst, &tmap_t, &S.full[s], (kt - kw_steps) * kBK, (int)m0);
                    }
                }
            }
            __syncwarp();
            issued = g + 1;
        }
        // drain: every issued load has landed before the CTA may exit (a
        // pair's loads complete on the even CTA's barriers: its MMA issuer
        // drains them, and the cluster barrier at the end holds both CTAs)
        if (leader && (!kPair || issuer)) {
            for (int g = issued - kStages < 0 ? 0 : issued - kStages; g < issued; ++g) {
                const int s = g % kStages;
                const uint32_t ph = (uint32_t)(g / kStages) & 1u;
                unsigned long long t0 = global_ns();
                while (!mbar_try_wait(&S.full[s], ph) && global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp == 1 && issuer) {
        // ---------------- MMA issuer ----------------
        // The whole warp runs the loop (its values stay warp-uniform); one
        // elected lane issues the MMAs and the commits.
        const bool leader = elect_one();
        bool any = false, stop = false;
        // Stage s: x tile at descriptor xdesc0 + (s * kXStageBytes) / 16
        // (the start-address field counts 16-byte units and the sum is
        // the stage's own address), weight k-step j at tensor-memory
        // column kACol + 32 (kSub s + j).  Unrolled over the stages, so
        // every offset is a constant and the issue loop stays short.
        const uint64_t xdesc0 = smem_desc_sw128(S.x[0]);
        for (int g0 = 0; !stop && g0 < kg_total; g0 += kStages) {
            const uint32_t ph = (uint32_t)(g0 / kStages) & 1u;
#pragma unroll
            for (int s = 0; s < kStages; ++s) {
                const int g = g0 + s;
                if (g >= kg_total) break;
                if (!__all_sync(0xFFFFFFFFu, mbar_wait<kPair>(&S.full[s], ph, abort, err))) {
                    stop = true;
                    break;
                }
                tc_fence_after();
                if (leader) {
#pragma unroll
                    for (int j = 0; j < kSub; ++j) {
                        const int i = g * kSub + j;
                        if (kSub == 1 || i < steps) {
                            const uint64_t bdesc = xdesc0 + (uint64_t)((s * kXStageBytes + j * kXSubBytes) >> 4);
                            const uint32_t acol = tmem + kACol + 32u * (uint32_t)(kSub * s + j);
                            // the first step of each segment starts its accumulator
                            const uint32_t dcol = tmem + kAccCol + C::AccCols * (uint32_t)seg_of(i);
                            if constexpr (kPair) {
                                tc_mma_ts_pair(dcol, acol, bdesc, C::Idesc, i != 0 ? 1u : 0u);
#pragma unroll
                                for (int kk = 1; kk < kBK / 16; ++kk)
                                    tc_mma_ts_pair(dcol, acol + 8u * kk, bdesc + 2ull * kk, C::Idesc, 1u);
                            } else {
                                tc_mma_ts(dcol, acol, bdesc, C::Idesc, (i != 0 && i != i_next) ? 1u : 0u);
#pragma unroll
                                for (int kk = 1; kk < kBK / 16; ++kk)
                                    tc_mma_ts(dcol, acol + 8u * kk, bdesc + 2ull * kk, C::Idesc, 1u);
                            }
                        }
                    }
                    // stage s is free again in both CTAs of a pair
                    if constexpr (kPair) {
                        tc_commit_pair(cluster_addr(&S.empty[s], 0));
                        tc_commit_pair(cluster_addr(&S.empty[s], 1));
                    } else {
                        tc_commit(&S.empty[s]);
                    }
                }
                __syncwarp();
                any = true;
            }
        }
        if (leader) {
            if (any && !stop) {
                if constexpr (kPair) {
                    tc_commit_pair(cluster_addr(&S.acc_full, 0));
                    tc_commit_pair(cluster_addr(&S.acc_full, 1));
                } else {
                    tc_commit(&S.acc_full);
                }
            }
            if (any && *abort) {  // drain our own MMAs before tensor memory is released
                if constexpr (kPair) tc_commit_pair(cluster_addr(&S.drain, 0));
                else tc_commit(&S.drain);
                unsigned long long t0 = global_ns();
                while (!mbar_try_wait(&S.drain, 0) && global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ---------------- dequant warpgroups, then epilogue ----------------
        const int q = warp & 3;         // tensor-memory lane quarter
        const int h = (warp - 4) >> 2;  // warpgroup: k-steps with index % kWG == h
        const int row_in_tile = 32 * q + lane;
        // weight row of step i (the next tile's from i_next on)
        auto row_of = [&](int i) { return n0 + (int64_t)kBN * seg_of(i) + row_in_tile; };
        const float mu = (kMode == 0) ? __ldg(offset) : 0.0f;
        const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
        bool ok = true;
        // software pipeline: the codes of this warpgroup's next kPF stages
        // (kSub k-steps each) are in flight while the current one is
        // converted.  The register sets form a ring of kPF + 1 stages,
        // indexed at compile time by unrolling kPF + 1 stages, so no set is
        // copied (a copy would wait for its load).
        constexpr int kPF = NF4_GEMM_PF;
        StepCodes ring[kPF + 1][kSub];
        auto load_group = [&](int g, StepCodes(&set)[kSub]) {
#pragma unroll
            for (int j = 0; j < kSub; ++j) {
                const int i = g * kSub + j;
                const int kt = kt_of(i);
                const int64_t n = row_of(i);
                if (i < steps && kt < kw_steps) load_step<kMode>(packed, q8, scales, mu, n, K, kt, n < N, set[j]);
            }
        };
#pragma unroll
        for (int i = 0; i < kPF; ++i) {
            const int g = h + i * kWG;
            if (g < kg_total) load_group(g, ring[i]);
        }
        for (int g0 = h; ok && g0 < kg_total; g0 += (kPF + 1) * kWG) {
#pragma unroll
            for (int i = 0; i <= kPF; ++i) {
                const int g = g0 + i * kWG;
                if (g >= kg_total) break;
                const int s = g % kStages;
                const uint32_t ph = (uint32_t)(g / kStages) & 1u;
                if (g + kPF * kWG < kg_total) load_group(g + kPF * kWG, ring[(i + kPF) % (kPF + 1)]);
#pragma unroll
                for (int j = 0; j < kSub; ++j) {
                    const int ii = g * kSub + j;
                    if (ii >= steps) break;
                    const int kt = kt_of(ii);
                    uint32_t v[32];
                    if (kt < kw_steps) {
                        if ((kLutMask >> h) & 1) dequant_step_smem<kMode>(ring[i][j], mu, S.pairs + (lane & 15), v);
                        else dequant_step<kMode>(ring[i][j], mu, v);
                    } else {
                        const int64_t n = row_of(ii);
                        lora_step(Bl, r, n, n < N, kt - kw_steps, v);
                    }
                    if (j == 0) {
                        // warp-uniform outcome: the tcgen05.st below is a warp-wide instruction
                        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&S.empty[s], ph ^ 1u, abort, err));
                        if (!ok) break;
                    }
                    tc_store32(lane_base + kACol + 32u * (uint32_t)(kSub * s + j), v);
                    tc_wait_st();
                }
                if (!ok) break;
                tc_fence_before();
                if constexpr (kPair) mbar_arrive_cluster(cluster_addr(&S.full[s], 0));
                else mbar_arrive(&S.full[s]);
            }
        }
        if (ok) ok = __all_sync(0xFFFFFFFFu, mbar_wait(&S.acc_full, 0, abort, err));
        if constexpr (kSK) {
            // Epilogue (stream-K): warpgroup h takes segment h.
            const int nseg = steps > i_next ? 2 : 1;
            if (h < nseg) {
                const int64_t tile = tile0 + h;
                if (ok) {
                    tc_fence_after();
                    uint32_t v[32];
                    tc_load32(lane_base + kAccCol + C::AccCols * (uint32_t)h, v);  // columns 16..31 unused
                    tc_wait_ld();
                    float *dst = partials + (int64_t)(2 * blockIdx.x + h) * kPartialFloats + row_in_tile;
#pragma unroll
                    for (int m = 0; m < 16; ++m) dst[m * 128] = __uint_as_float(v[m]);
                }
                __threadfence();  // the partial is visible before this CTA's arrival
                asm volatile("bar.sync %0, 128;" ::"r"(2 + h) : "memory");
                if (row_in_tile == 0) {
                    // the counts were zeroed by the grid before this one
                    asm volatile("griddepcontrol.wait;" ::: "memory");
                    const int64_t c0 = nf4_sk_owner(tile * kt_total, total, gridDim.x);
                    const int64_t c1 = nf4_sk_owner(tile * kt_total + kt_total - 1, total, gridDim.x);
                    const unsigned prev = atomicAdd(counts + tile, 1u);
                    S.last[h] = prev == (unsigned)(c1 - c0);
                }
                asm volatile("bar.sync %0, 128;" ::"r"(2 + h) : "memory");
                if (S.last[h]) {
                    // every partial of the tile is in: add them in CTA order
                    __threadfence();
                    const int64_t c0 = nf4_sk_owner(tile * kt_total, total, gridDim.x);
                    const int64_t c1 = nf4_sk_owner(tile * kt_total + kt_total - 1, total, gridDim.x);
                    float acc[16];
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc[m] = 0.0f;
                    for (int64_t c = c0; c <= c1; ++c) {
                        // segment 0 when CTA c's range starts in this tile, else 1
                        const int seg = nf4_sk_segment(c, tile, kt_total, total, gridDim.x);
                        const float *src = partials + (2 * c + seg) * kPartialFloats + row_in_tile;
#pragma unroll
                        for (int m = 0; m < 16; ++m) acc[m] += __ldcg(src + m * 128);
                    }
                    const int64_t n = tile * kBN + row_in_tile;
                    if (n < N) {
#pragma unroll
                        for (int m = 0; m < 16; ++m)
                            if (m < M) y[m * N + n] = __float2bfloat16_rn(acc[m]);
                    }
                }
            }
        } else if (ok) {
            // Epilogue: accumulators -> bf16 -> staging tile Y[m][n] (256 x 128,
            // row-major, in the now idle x ring) -> one TMA store, which also
            // clips rows and columns outside y.
            tc_fence_after();
            __nv_bfloat16 *stage = reinterpret_cast<__nv_bfloat16 *>(&S.x[0][0]);
#pragma unroll 1
            for (int c = h; c < (kBT + 31) / 32; c += kWG) {  // 32-token chunks of the tile
                uint32_t v[32];
                tc_load32(lane_base + kAccCol + 32u * c, v);  // the allocation holds >= 32 columns
                tc_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (32 * c + i < kBT)
                        stage[(32 * c + i) * kBN + row_in_tile] = __float2bfloat16_rn(__uint_as_float(v[i]));
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        // all dequant/epilogue threads have staged their values (or given up)
        asm volatile("bar.sync 1, %0;" ::"n"(128 * kWG) : "memory");
        if (!kSK && threadIdx.x == 128 && !*abort) {
            asm volatile(
                "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                    reinterpret_cast<uint64_t>(&tmap_y)),
                "r"((int)n0), "r"((int)m0), "r"(smem_addr(&S.x[0][0]))
                : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        }
    }
    tc_fence_before();
    __syncthreads();
    // a pair: neither CTA releases its tensor memory (read by the pair's
    // MMAs) or leaves (its shared memory is the pair's B operand) before the other is done
    if constexpr (kPair) cluster_sync_all();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        if constexpr (kPair)
            asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
        else
            asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

template <int kMode, class C, bool kSK>
cudaError_t launch_mode(const CUtensorMap &mx, const CUtensorMap &mt, const CUtensorMap &my, int64_t M, int64_t K, int64_t N,
                        const uint8_t *packed, const uint8_t *q8, const float *scales, const float *offset,
                        const __nv_bfloat16 *Bl, int r, int rp, __nv_bfloat16 *y, float *partials, unsigned *counts,
                        int ctas, unsigned *err, cudaStream_t stream) {
    const size_t smem = sizeof(SmemLayout<C>) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(k_gemm_tc<kMode, C, kSK>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    int64_t tiles = (N + kBN - 1) / kBN;
    if (C::Pair) tiles = (tiles + 1) & ~(int64_t)1;  // whole pairs (a last odd tile's partner has no rows)
    cfg.gridDim = kSK ? dim3((unsigned)ctas) : dim3((unsigned)tiles, (unsigned)((M + C::BT - 1) / C::BT));
    cfg.blockDim = dim3(C::Threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = C::Pair ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k_gemm_tc<kMode, C, kSK>, mx, mt, my, M, K, N, packed, q8, scales, offset, Bl, r,
                              rp, y, partials, counts, err);
}

template <class C, bool kSK>
cudaError_t launch_cfg(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                       const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                       void *y, float *partials, unsigned *counts, int ctas, cudaStream_t stream,
                       unsigned *err_word) {
    CUtensorMap mx, mt, my;
    cudaError_t e = make_map(&mx, x, M, K, kBK, C::XRows, true);
    if (e != cudaSuccess) return e;
    if (r > 0) e = make_map(&mt, t2, M, rp, kBK, C::XRows, true);
    else e = make_map(&mt, x, M, K, kBK, C::XRows, true);  // unused: no extension steps
    if (e != cudaSuccess) return e;
    e = make_map(&my, y, M, N, kBN, C::BT, false);
    if (e != cudaSuccess) return e;
    auto *Bl = static_cast<const __nv_bfloat16 *>(B);
    auto *yp = static_cast<__nv_bfloat16 *>(y);
    if (q8 == nullptr)
        return launch_mode<2, C, kSK>(mx, mt, my, M, K, N, packed, q8, scales, offset, Bl, r, rp, yp, partials, counts,
                                      ctas, err_word, stream);
    if (offset == nullptr)
        return launch_mode<1, C, kSK>(mx, mt, my, M, K, N, packed, q8, scales, offset, Bl, r, rp, yp, partials, counts,
                                      ctas, err_word, stream);
    return launch_mode<0, C, kSK>(mx, mt, my, M, K, N, packed, q8, scales, offset, Bl, r, rp, yp, partials, counts,
                                  ctas, err_word, stream);
}

// ---------------------------------------------------------------------------
// LoRA down-projection for large M on the tensor cores:
//   t = s x A^T,  x [M, K] bf16,  A [r, K] bf16,  t as [t_hi | t_lo | 0] bf16
// (same output as the warp-MMA kernel in lora_down.cu).  A thread-block
// cluster of kSplit CTAs (1, 2 or 4) owns 128 rows of x and splits K: CTA c runs the
// k-steps [c kt / kSplit, (c + 1) kt / kSplit) as
// D[128, r] += X[128, k] A[r, k]^T with both operands brought by TMA (128-byte
// swizzle, kDownStages-deep ring) and one thread issuing the MMAs (M = 128,
// N = r, K = 16) into r fp32 columns of its tensor memory.  Each CTA then
// stages its partial tile in shared memory, and CTA c finishes rows
// [128 c / kSplit, 128 (c + 1) / kSplit) of the tile: it adds the
// kSplit partials in rank order
// through distributed shared memory (so the result does not depend on
// timing), scales, and writes the hi/lo pair.
// The kernel runs alongside the fused GEMM (programmatic dependent launch),
// so what it costs the GEMM is SMs x time: one CTA per 128 rows with a deep
// ring (no split) takes the fewest SM-microseconds; splitting K over a
// cluster shortens the kernel but holds more SMs.
#ifndef NF4_DOWN_STAGES
#define NF4_DOWN_STAGES 8
#endif
#ifndef NF4_DOWN_SPLIT
#define NF4_DOWN_SPLIT 1
#endif
constexpr int kDownStages = NF4_DOWN_STAGES;
constexpr int kDownRows = 128;
constexpr int kDownSplit = NF4_DOWN_SPLIT;  // default cluster size along K

template <int kR>
struct __align__(1024) DownSmem {
    uint8_t x[kDownStages][kDownRows * 128];  // after the main loop: the fp32 partial tile [kR][128]
    uint8_t a[kDownStages][kR * 128];
    uint64_t full[kDownStages];
    uint64_t empty[kDownStages];
    uint64_t acc_full;
    uint32_t tmem_base;
    int abort;
};
static_assert(kDownStages * kDownRows * 128 >= 64 * kDownRows * 4, "partial tile fits in the x ring");

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

template <int kR, int kSplit>
__global__ void __launch_bounds__(128, 1)
    k_lora_down_tc(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_a, int64_t M,
                   int64_t K, float scaling, __nv_bfloat16 *__restrict__ t2, int rp, unsigned *err) {
    constexpr uint32_t kCols = kR < 32 ? 32 : kR;  // tensor memory allocation (power of 2, >= 32)
    constexpr uint32_t kIdescDown = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kR >> 3) << 17) |
                                    ((uint32_t)(kDownRows >> 4) << 24);
    constexpr uint32_t kStageBytes = kDownRows * 128 + kR * 128;
    extern __shared__ uint8_t smem_raw[];
    DownSmem<kR> &S =
        *reinterpret_cast<DownSmem<kR> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int *abort = &S.abort;
    // the fused linear launched next may start once every CTA is past this
    // point; it reads x and W at once and waits for t itself
    pdl_wait_then_release();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int64_t m0 = (int64_t)blockIdx.y * kDownRows;
    const int kt_all = (int)((K + 63) / 64);  // a partial last step reads zeros beyond K (TMA fill)
    const int kt_begin = (int)((int64_t)rank * kt_all / kSplit);
    const int kt_total = (int)((int64_t)(rank + 1) * kt_all / kSplit) - kt_begin;
    if (threadIdx.x == 0) {
        for (int st = 0; st < kDownStages; ++st) {
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
                     "r"(kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    bool ok = true;
    if (threadIdx.x == 0 && kt_total > 0) {
        // producer: the x and A boxes of every k-step, kDownStages ahead of the MMAs
        int issued = 0;
        for (; issued < kt_total; ++issued) {
            const int st = issued % kDownStages;
            const uint32_t ph = (uint32_t)(issued / kDownStages) & 1u;
            if (!mbar_wait(&S.empty[st], ph ^ 1u, abort, err)) break;
            mbar_arrive_expect_tx(&S.full[st], kStageBytes);
            tma_load_2d(S.x[st], &tmap_x, &S.full[st], (kt_begin + issued) * 64, (int)m0);
            tma_load_2d(S.a[st], &tmap_a, &S.full[st], (kt_begin + issued) * 64, 0);
        }
        if (*abort) {  // every issued load lands before the CTA may exit
            for (int kt = issued - kDownStages < 0 ? 0 : issued - kDownStages; kt < issued; ++kt) {
                unsigned long long t0 = global_ns();
                while (!mbar_try_wait(&S.full[kt % kDownStages], (uint32_t)(kt / kDownStages) & 1u) &&
                       global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
    } else if (threadIdx.x == 32 && kt_total > 0) {
        // MMA issuer (its own thread, so that the loads and the MMAs of
        // consecutive k-steps overlap): D[128 rows, r] += x A^T per k-step
        for (int kt = 0; kt < kt_total; ++kt) {
            const int st = kt % kDownStages;
            if (!mbar_wait(&S.full[st], (uint32_t)(kt / kDownStages) & 1u, abort, err)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint64_t ad = smem_desc_sw128(S.x[st]), bd = smem_desc_sw128(S.a[st]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                tc_mma_ss(tmem, ad + 2ull * kk, bd + 2ull * kk, kIdescDown, (kt | kk) != 0 ? 1u : 0u);
            tc_commit(&S.empty[st]);
        }
        tc_commit(&S.acc_full);
    }
    __syncwarp();
    // this CTA's partial tile -> shared memory, column-major [kR][128] fp32
    // (the x ring is free: every MMA that read it has completed)
    float *part = reinterpret_cast<float *>(&S.x[0][0]);
    const int row = 32 * warp + lane;  // tensor-memory lane = tile row
    if (kt_total > 0) {
        if (__all_sync(0xFFFFFFFFu, mbar_wait(&S.acc_full, 0, abort, err))) {
            tc_fence_after();
            const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16);
#pragma unroll
            for (int c0 = 0; c0 < (int)kCols; c0 += 32) {
                uint32_t v[32];
                tc_load32(taddr + (uint32_t)c0, v);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (c0 + j < kR) part[(c0 + j) * kDownRows + row] = __uint_as_float(v[j]);
            }
        }
    } else {
        for (int c = 0; c < kR; ++c) part[c * kDownRows + row] = 0.0f;  // no k-steps: a zero partial
    }
    cluster_sync_all();  // every CTA's partial is complete and visible in the cluster
    // finish rows [kRowsPer rank, kRowsPer (rank + 1)): thread t takes row
    // kRowsPer rank + t % kRowsPer and the kCw columns of group t / kRowsPer
    {
        constexpr int kRowsPer = kDownRows / kSplit;
        constexpr int kCw = kR / (128 / kRowsPer);  // columns per thread (>= 4)
        static_assert(kCw % 4 == 0, "whole 4-column chunks");
        const int t = threadIdx.x;
        const int r_loc = kRowsPer * (int)rank + t % kRowsPer;
        const int64_t m = m0 + r_loc;
        const int cb = (t / kRowsPer) * kCw;
        uint32_t base[kSplit];
#pragma unroll
        for (int c = 0; c < kSplit; ++c) base[c] = cluster_addr(part + cb * kDownRows + r_loc, (uint32_t)c);
#pragma unroll 1
        for (int j0 = 0; j0 < kCw; j0 += 4) {
            float v[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float a = 0.0f;
#pragma unroll
                for (int c = 0; c < kSplit; ++c)
                    a += ld_cluster_f32(base[c] + (uint32_t)((j0 + j) * kDownRows * 4));
                v[j] = a * scaling;
            }
            if (m < M) {
                uint32_t hi[2], lo[2];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const __nv_bfloat16 h0 = __float2bfloat16_rn(v[2 * j]), h1 = __float2bfloat16_rn(v[2 * j + 1]);
                    hi[j] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
                    lo[j] = pack_bf16x2(v[2 * j] - __bfloat162float(h0), v[2 * j + 1] - __bfloat162float(h1));
                }
                *reinterpret_cast<uint2 *>(t2 + m * rp + cb + j0) = make_uint2(hi[0], hi[1]);
                *reinterpret_cast<uint2 *>(t2 + m * rp + kR + cb + j0) = make_uint2(lo[0], lo[1]);
            }
        }
        if (m < M && cb == 0)
            for (int j = 2 * kR; j < rp; j += 8)
                *reinterpret_cast<uint4 *>(t2 + m * rp + j) = make_uint4(0u, 0u, 0u, 0u);
    }
    cluster_sync_all();  // no CTA leaves while another may still read its partial
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols) : "memory");
    }
}

// Persistent form without a K split (the default alongside the fused GEMM):
// CTA c takes the 128-row tiles c, c + gridDim.x, ..., so the launch can be
// held to the SMs the GEMM leaves idle.  Warp 4 (one lane) streams the x and
// A boxes of every tile through the ring, warp 5 (one lane) issues the MMAs
// into one of two tensor-memory accumulators (tile parity), and warps 0-3
// (tensor-memory lane quarters) turn each finished accumulator into rows of
// t while the next tile's MMAs run.
constexpr int kDownPThreads = 192;

template <int kR>
struct __align__(1024) DownPSmem {
    uint8_t x[kDownStages][kDownRows * 128];
    uint8_t a[kDownStages][kR * 128];
    uint64_t full[kDownStages];
    uint64_t empty[kDownStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint32_t tmem_base;
    int abort;
};

template <int kR>
__global__ void __launch_bounds__(kDownPThreads, 1)
    k_lora_down_tc_p(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_a,
                     int64_t M, int64_t K, float scaling, __nv_bfloat16 *__restrict__ t2, int rp, unsigned *err) {
    constexpr uint32_t kCols = kR < 32 ? 32 : kR;  // one accumulator; two are allocated
    constexpr uint32_t kIdescDown = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kR >> 3) << 17) |
                                    ((uint32_t)(kDownRows >> 4) << 24);
    constexpr uint32_t kStageBytes = kDownRows * 128 + kR * 128;
    extern __shared__ uint8_t smem_raw[];
    DownPSmem<kR> &S =
        *reinterpret_cast<DownPSmem<kR> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    volatile int *abort = &S.abort;
    // the fused linear launched next may start once every CTA is past this
    // point; it reads x and W at once and waits for t itself
    pdl_wait_then_release();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = (int)((M + kDownRows - 1) / kDownRows);
    const int kt_total = (int)((K + 63) / 64);  // a partial last step reads zeros beyond K (TMA fill)
    if (threadIdx.x == 0) {
        for (int st = 0; st < kDownStages; ++st) {
            mbar_init(&S.full[st], 1);
            mbar_init(&S.empty[st], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&S.acc_full[b], 1);
            mbar_init(&S.acc_empty[b], 4);
        }
        S.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&S.tmem_base)),
                     "r"(2 * kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = S.tmem_base;

    if (warp == 4) {
        if (lane == 0) {
            // producer: every k-step of every tile, kDownStages ahead of the MMAs
            int64_t g = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
                for (int kt = 0; kt < kt_total; ++kt, ++g) {
                    const int st = (int)(g % kDownStages);
                    const uint32_t ph = (uint32_t)(g / kDownStages) & 1u;
                    if (!mbar_wait(&S.empty[st], ph ^ 1u, abort, err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&S.full[st], kStageBytes);
                    tma_load_2d(S.x[st], &tmap_x, &S.full[st], kt * 64, tile * kDownRows);
                    tma_load_2d(S.a[st], &tmap_a, &S.full[st], kt * 64, 0);
                }
            }
            if (*abort) {  // every issued load lands before the CTA may exit
                for (int64_t k2 = g - kDownStages < 0 ? 0 : g - kDownStages; k2 < g; ++k2) {
                    const unsigned long long t0 = global_ns();
                    while (!mbar_try_wait(&S.full[k2 % kDownStages], (uint32_t)(k2 / kDownStages) & 1u) &&
                           global_ns() - t0 < kWaitLimitNs) {
                    }
                }
            }
        }
    } else if (warp == 5) {
        if (lane == 0) {
            // MMA issuer: D_b[128 rows, r] = x A^T of one tile, b = tile parity
            int64_t g = 0;
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
                const int b = it & 1;
                // the accumulator's previous tile has been read out
                if (it >= 2 && !mbar_wait(&S.acc_empty[b], (uint32_t)((it >> 1) - 1) & 1u, abort, err)) break;
                tc_fence_after();
                const uint32_t acc = tmem + (uint32_t)b * kCols;
                for (int kt = 0; kt < kt_total; ++kt, ++g) {
                    const int st = (int)(g % kDownStages);
                    if (!mbar_wait(&S.full[st], (uint32_t)(g / kDownStages) & 1u, abort, err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t ad = smem_desc_sw128(S.x[st]), bd = smem_desc_sw128(S.a[st]);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_ss(acc, ad + 2ull * kk, bd + 2ull * kk, kIdescDown, (kt | kk) != 0 ? 1u : 0u);
                    tc_commit(&S.empty[st]);
                }
                tc_commit(&S.acc_full[b]);
            }
        }
    } else {
        // epilogue: thread = tile row 32 warp + lane = tensor-memory lane
        int it = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
            const int b = it & 1;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&S.acc_full[b], (uint32_t)(it >> 1) & 1u, abort, err))) break;
            tc_fence_after();
            const int64_t m = (int64_t)tile * kDownRows + 32 * warp + lane;
            const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16) + (uint32_t)b * kCols;
#pragma unroll
            for (int c0 = 0; c0 < kR; c0 += 32) {
                uint32_t v[32];
                tc_load32(taddr + (uint32_t)c0, v);
                tc_wait_ld();
                if (m < M) {
                    const int kW = kR - c0 < 32 ? kR - c0 : 32;  // valid columns of this chunk
#pragma unroll
                    for (int j0 = 0; j0 < kW; j0 += 8) {
                        uint32_t hi[4], lo[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float v0 = __uint_as_float(v[j0 + 2 * j]) * scaling;
                            const float v1 = __uint_as_float(v[j0 + 2 * j + 1]) * scaling;
                            const __nv_bfloat16 h0 = __float2bfloat16_rn(v0), h1 = __float2bfloat16_rn(v1);
                            hi[j] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
                            lo[j] = pack_bf16x2(v0 - __bfloat162float(h0), v1 - __bfloat162float(h1));
                        }
                        *reinterpret_cast<uint4 *>(t2 + m * rp + c0 + j0) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                        *reinterpret_cast<uint4 *>(t2 + m * rp + kR + c0 + j0) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                }
            }
            if (m < M)
                for (int j = 2 * kR; j < rp; j += 8)
                    *reinterpret_cast<uint4 *>(t2 + m * rp + j) = make_uint4(0u, 0u, 0u, 0u);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.acc_empty[b]);  // the accumulator may be reused
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kCols) : "memory");
    }
}

template <int kR>
cudaError_t launch_down_tc_p(const CUtensorMap &mx, const CUtensorMap &ma, int64_t M, int64_t K, float s, void *t2,
                             int rp, unsigned *err, cudaStream_t stream, int max_ctas) {
    const size_t smem = sizeof(DownPSmem<kR>) + 1024;
    cudaError_t e =
        cudaFuncSetAttribute(k_lora_down_tc_p<kR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (M + kDownRows - 1) / kDownRows;
    const int64_t grid = max_ctas > 0 && max_ctas < tiles ? max_ctas : tiles;
    return launch_pdl(k_lora_down_tc_p<kR>, dim3((unsigned)grid), dim3(kDownPThreads), smem, stream, 1u, mx, ma, M,
                      K, s, static_cast<__nv_bfloat16 *>(t2), rp, err);
}

template <int kR, int kSplit>
cudaError_t launch_down_tc(const CUtensorMap &mx, const CUtensorMap &ma, int64_t M, int64_t K, float s, void *t2,
                           int rp, unsigned *err, cudaStream_t stream) {
    static_assert(kSplit == 1 || kSplit == 2 || kSplit == 4, "128 rows split evenly over the cluster");
    const size_t smem = sizeof(DownSmem<kR>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(k_lora_down_tc<kR, kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(k_lora_down_tc<kR, kSplit>, dim3(kSplit, (unsigned)((M + kDownRows - 1) / kDownRows)),
                      dim3(128), smem, stream, (unsigned)kSplit, mx, ma, M, K, s, static_cast<__nv_bfloat16 *>(t2), rp,
                      err);
}

template <int kR>
cudaError_t launch_down_tc_split(const CUtensorMap &mx, const CUtensorMap &ma, int64_t M, int64_t K, float s,
                                 void *t2, int rp, unsigned *err, cudaStream_t stream, int split, int max_ctas) {
    if (split == 4) return launch_down_tc<kR, 4>(mx, ma, M, K, s, t2, rp, err, stream);
    if (kDownSplit != 1) return launch_down_tc<kR, kDownSplit>(mx, ma, M, K, s, t2, rp, err, stream);
    return launch_down_tc_p<kR>(mx, ma, M, K, s, t2, rp, err, stream, max_ctas);
}

}  // namespace

// Scratch of a split launch: the partial tiles (2 per CTA) and one arrival
// count per weight tile.
int64_t streamk_partials_bytes() { return (int64_t)kStreamKMaxCtas * 2 * kPartialFloats * (int64_t)sizeof(float); }
int64_t streamk_counts_bytes() { return (int64_t)kStreamKMaxCtas * (int64_t)sizeof(unsigned); }

// CTAs of a split launch of the 16-token tile (0 = run it unsplit): `sms`
// SMs for the linear, at most kStreamKMaxCtas, none with fewer than
// kStreamKMinSteps k-steps, and more CTAs than 128-row tiles.
int streamk_ctas(int64_t M, int64_t K, int64_t N, int rp, int sms) {
    if (M > CfgSmall::BT) return 0;
    const int64_t ntiles = (N + kBN - 1) / kBN;
    const int64_t total = ntiles * (K / kBK + rp / kBK);
    int64_t ctas = sms < kStreamKMaxCtas ? sms : kStreamKMaxCtas;
    if (ctas > total / kStreamKMinSteps) ctas = total / kStreamKMinSteps;
    return ctas > ntiles ? (int)ctas : 0;
}

// ctas > 0 (from streamk_ctas): the split launch, with partials and counts
// from the caller's workspace (counts zeroed by the kernel launched just
// before); otherwise one CTA per tile.
cudaError_t launch_gemm_tc(const void *x, int64_t M, int64_t K, int64_t N, const uint8_t *packed, const uint8_t *q8,
                           const float *scales, const float *offset, const void *B, int r, const void *t2, int rp,
                           void *y, float *partials, unsigned *counts, int ctas, cudaStream_t stream,
                           unsigned *err_word) {
    if (M > 0x7FFFFFFF || K > 0x7FFFFFFF) return cudaErrorInvalidValue;
    if (M <= CfgSmall::BT) {
        if (ctas > 0)
            return launch_cfg<CfgSmall, true>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, partials,
                                              counts, ctas, stream, err_word);
        return launch_cfg<CfgSmall, false>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, nullptr, nullptr,
                                           0, stream, err_word);
    }
    if (NF4_GEMM_PAIR)
        return launch_cfg<CfgPair, false>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, nullptr, nullptr,
                                          0, stream, err_word);
    return launch_cfg<CfgLarge, false>(x, M, K, N, packed, q8, scales, offset, B, r, t2, rp, y, nullptr, nullptr, 0,
                                       stream, err_word);
}

// Tensor-core LoRA down-projection: see k_lora_down_tc.  split: 0 = the
// default (persistent CTAs over the 128-row tiles, the least SM time while a
// fused GEMM runs alongside; max_ctas > 0 caps the grid, e.g. to the SMs the
// GEMM leaves idle); 4 = K split over a 4-CTA cluster (a long contraction
// with nothing running alongside).
cudaError_t launch_lora_down_tc(const void *x, const void *A, int64_t M, int64_t K, int r, float s, void *t2, int rp,
                                unsigned *err, cudaStream_t stream, int split, int max_ctas) {
    if (M > 0x7FFFFFFF || K > 0x7FFFFFFF) return cudaErrorInvalidValue;
    CUtensorMap mx, ma;
    cudaError_t e = make_map(&mx, x, M, K, 64, kDownRows, true);
    if (e != cudaSuccess) return e;
    e = make_map(&ma, A, r, K, 64, r, true);
    if (e != cudaSuccess) return e;
    switch (r) {
        case 16: return launch_down_tc_split<16>(mx, ma, M, K, s, t2, rp, err, stream, split, max_ctas);
        case 32: return launch_down_tc_split<32>(mx, ma, M, K, s, t2, rp, err, stream, split, max_ctas);
        case 64: return launch_down_tc_split<64>(mx, ma, M, K, s, t2, rp, err, stream, split, max_ctas);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace nf4
