/*
 * nf4.h -- C ABI of libnf4.so: QLoRA NF4 blockwise weight quantization with
 * double quantization, dequantization and the fused frozen-base LoRA linear,
 * on one NVIDIA B200 (sm_100a).
 *
 * Sources (web pages, cited by title and section):
 *   [MF]  "QLoRA: Mathematical Foundations of 4-Bit NormalFloat Quantization,
 *         Double Quantization, and Paged Optimizers" (llms.blog)
 *   [L15] "Lesson 15. NF4 and Double Quantisation" (tokencemetery)
 *   [AD]  "QLoRA: quantising the part you are not training" (addaly.com)
 *   [QP]  "QLoRA in Production: 4-bit NormalFloat & Double Quantization Deep
 *         Dive" (devtechtools.org)
 *
 * Conventions for every entry point
 *   - Device buffers are allocated and owned by the caller; the library never
 *     allocates or frees device memory.  Pointers marked "device" must point
 *     to memory of the current CUDA device; "host" pointers to host memory.
 *   - Device pointers must be 16-byte aligned (NF4_ERR_INVALID otherwise).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls only enqueue work: they return once the kernels are
 *     launched, and results are valid after the stream is synchronized.
 *   - Sizes are element counts unless named *_bytes.
 *   - Inputs must be finite (not checked).
 *   - Return value: NF4_OK, NF4_ERR_INVALID (bad pointer, size or alignment;
 *     nothing was launched), NF4_ERR_UNSUPPORTED (a block size or rank this
 *     build does not implement; nothing was launched), NF4_ERR_CUDA (a CUDA
 *     launch or runtime error; see nf4_last_cuda_error), NF4_ERR_TIMEOUT
 *     (reported only by nf4_device_status: a bounded wait inside a kernel
 *     expired and the kernel returned early; its outputs are invalid).
 *
 * Data layout (READINGS of what the pages leave open are marked):
 *   - A weight W[N, K] (PyTorch Linear layout, row n = output feature n) is
 *     flattened row-major, n = N*K elements, and cut into contiguous blocks of
 *     64 ([MF] "Block-Wise Quantization Mechanics"; the last block may be
 *     shorter).  nblocks = ceil(n / 64).
 *   - packed: uint8[n/2]; READING: element 2j in the high nibble of byte j,
 *     element 2j+1 in the low nibble.  Codes index the NF4 table.
 *   - absmax: fp32[nblocks], c1 = max |w| of each block.
 *   - Double quantization ([MF] "Double Quantization (DQ)"): absmax_q
 *     uint8[nblocks] holds OCP FP8 E4M3 codes (READING of "FP8") of
 *     (c1 - mu) / c2; absmax2 fp32[ceil(nblocks / 256)] holds c2 per run of
 *     256 constants; offset fp32[1] holds mu, one per tensor (READING of the
 *     "bias/mean subtraction"; NULL offset = no centring, mu = 0).
 *   - Storage per parameter: 0.5 + 1/64 + 4/16384 bytes ([L15] "Double
 *     quantisation"), plus 4 bytes of offset per tensor.
 */
#ifndef NF4_H_
#define NF4_H_

#include <stdint.h>

#if defined(__GNUC__)
#define NF4_API __attribute__((visibility("default")))
#else
#define NF4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NF4_OK = 0,
    NF4_ERR_INVALID = 1,
    NF4_ERR_UNSUPPORTED = 2,
    NF4_ERR_CUDA = 3,
    NF4_ERR_TIMEOUT = 4
} nf4_status;

typedef enum { NF4_F32 = 0, NF4_BF16 = 1 } nf4_dtype;

/* Human-readable name of a status code (static string). */
NF4_API const char *nf4_status_string(nf4_status s);

/* The last CUDA error code (cudaError_t as int) seen by a call that
 * returned NF4_ERR_CUDA in this process; 0 if none. */
NF4_API int nf4_last_cuda_error(void);

/* nf4_codebook -- the sixteen NF4 levels q_0..q_15 ([MF] section "4-Bit
 * NormalFloat (NF4)", the printed list: q_0 = -1, q_7 = 0, q_15 = 1).
 * out_host: host float[16], written in index order.  NF4_ERR_INVALID if
 * NULL.  Pure host call; no device work. */
NF4_API nf4_status nf4_codebook(float *out_host);

/* nf4_quantize -- blockwise NF4 quantization ([MF] "Block-Wise Quantization
 * Mechanics": c1 = max_j |w_j| per contiguous block of 64, code_j = arg-min_i
 * |w_j / c1 - q_i|).  The quotient w_j / c1 is the IEEE binary32 quotient;
 * READING: exact ties go to the lower index; an all-zero block gives c1 = 0
 * and code 7 (the exact zero) for every element.
 *   w        device, n elements of w_dtype (NF4_F32 or NF4_BF16)
 *   n        element count, even, >= 0
 *   blocksize must be 64 (else NF4_ERR_UNSUPPORTED)
 *   packed   device uint8[n/2]  (output)
 *   absmax   device fp32[ceil(n/64)]  (output)
 * One kernel launch. */
NF4_API nf4_status nf4_quantize(const void *w, nf4_dtype w_dtype, int64_t n, int blocksize,
                        uint8_t *packed, float *absmax, void *stream);

/* Bytes of device workspace nf4_quantize_dq needs for n weights (the fp32
 * block constants, then the fp64 run sums of the centring mean); 0 for
 * n <= 0 or unsupported block sizes. */
NF4_API int64_t nf4_quantize_dq_workspace_size(int64_t n, int blocksize, int dq_blocksize);

/* nf4_quantize_dq -- nf4_quantize followed by nf4_double_quantize in one call
 * ([MF] "Block-Wise Quantization Mechanics" and "Double Quantization (DQ)"):
 * the stored format straight from the weight.  Every output is bit-identical
 * to the two calls made in turn; the fp32 constants only pass through the
 * workspace.
 *   w          device, n elements of w_dtype; n even, >= 0
 *   blocksize 64, dq_blocksize 256 (else NF4_ERR_UNSUPPORTED)
 *   packed     device uint8[n/2]            (output)
 *   absmax_q   device uint8[ceil(n/64)]     (output)
 *   absmax2    device fp32[ceil(n/16384)]   (output)
 *   offset     device fp32[1] (output mu) or NULL (no centring)
 *   workspace  device scratch, 256-byte aligned, workspace_bytes >=
 *              nf4_quantize_dq_workspace_size(n, 64, 256); contents on entry
 *              are ignored.
 * Three kernel launches with centring (four above 2048 runs, i.e. 33.5 M
 * weights), two without. */
NF4_API nf4_status nf4_quantize_dq(const void *w, nf4_dtype w_dtype, int64_t n, int blocksize, int dq_blocksize,
                                   uint8_t *packed, uint8_t *absmax_q, float *absmax2, float *offset,
                                   void *workspace, int64_t workspace_bytes, void *stream);

/* Bytes of device workspace nf4_double_quantize needs for nblocks first-level
 * constants with centring (0 when nblocks == 0). */
NF4_API int64_t nf4_double_quantize_workspace_size(int64_t nblocks, int dq_blocksize);

/* nf4_double_quantize -- quantize the fp32 block constants to 8 bits in runs
 * of 256, each run with an fp32 second-level scale ([MF] "Double Quantization
 * (DQ)": c2 = max |c1| per run, c1_FP8 = quantize_FP8(c1 / c2)).
 * READINGS: the 8-bit format is OCP FP8 E4M3, round to nearest even,
 * saturating; with `offset` non-NULL one per-tensor mean mu is subtracted
 * first (c2 = max |c1 - mu|, code = E4M3((c1 - mu) / c2), each step one
 * binary32 rounding), where mu = RN_f32(S / nblocks) and S is a fixed-order
 * binary64 sum: each run of 256 summed in index order, then the run sums
 * combined pairwise level by level (an odd last element carried up).  A run
 * with c2 = 0 stores code 0.
 *   absmax     device fp32[nblocks]   (input, from nf4_quantize)
 *   nblocks    >= 0
 *   dq_blocksize must be 256 (else NF4_ERR_UNSUPPORTED)
 *   absmax_q   device uint8[nblocks]  (output)
 *   absmax2    device fp32[ceil(nblocks/256)]  (output)
 *   offset     device fp32[1] (output mu) or NULL (no centring)
 *   workspace  device scratch of workspace_bytes >=
 *              nf4_double_quantize_workspace_size(); may be NULL when offset
 *              is NULL.  Contents on entry are ignored; the caller keeps
 *              ownership; it must not be used by other work until the
 *              stream passes this call.
 * Two kernel launches with centring (three above 2048 runs), one without. */
NF4_API nf4_status nf4_double_quantize(const float *absmax, int64_t nblocks, int dq_blocksize,
                               uint8_t *absmax_q, float *absmax2, float *offset,
                               void *workspace, int64_t workspace_bytes, void *stream);

/* nf4_dq_run_sums -- the first step of the centring mean of nf4_double_quantize
 * on its own: run_sums[d] = the binary64 sum of the constants of run d (256
 * consecutive constants, the last run possibly shorter), summed in index
 * order ([MF] "Double Quantization (DQ)": the per-tensor "bias/mean
 * subtraction"; the summation order is the READING stated for
 * nf4_double_quantize).  For a tensor split over ranks on run boundaries
 * (every shard but the last a multiple of 16,384 weights) each rank computes
 * its runs' sums; the caller gathers them in shard order and passes the whole
 * array to nf4_double_quantize_sharded.
 *   absmax    device fp32[nblocks]  (this shard's constants, from nf4_quantize)
 *   run_sums  device fp64[ceil(nblocks / 256)]  (output)
 * NF4_ERR_UNSUPPORTED if dq_blocksize != 256.  One kernel launch. */
NF4_API nf4_status nf4_dq_run_sums(const float *absmax, int64_t nblocks, int dq_blocksize, double *run_sums,
                                   void *stream);

/* Bytes of device workspace nf4_double_quantize_sharded needs for a tensor
 * of nblocks_total constants. */
NF4_API int64_t nf4_double_quantize_sharded_workspace_size(int64_t nblocks_total, int dq_blocksize);

/* nf4_double_quantize_sharded -- nf4_double_quantize (with centring) of one
 * shard of a tensor, with the mean of the whole tensor: mu = RN_f32(S /
 * nblocks_total), S the fixed pairwise tree over the run sums of ALL runs of
 * the tensor (run_sums_all, as written by nf4_dq_run_sums on every shard and
 * concatenated in shard order).  Codes, c2 and mu are bit-identical to
 * nf4_double_quantize of the whole tensor, for any split on run boundaries.
 *   absmax        device fp32[nblocks], this shard's constants (0 allowed:
 *                 only mu is written)
 *   run_sums_all  device fp64[ceil(nblocks_total / 256)]
 *   absmax_q      device uint8[nblocks]; absmax2 device fp32[ceil(nblocks/256)]
 *   offset        device fp32[1] (output mu; required)
 *   workspace     device scratch, workspace_bytes >=
 *                 nf4_double_quantize_sharded_workspace_size(nblocks_total)
 * NF4_ERR_INVALID for nblocks > nblocks_total or missing buffers.  Two kernel
 * launches (one when nblocks == 0). */
NF4_API nf4_status nf4_double_quantize_sharded(const float *absmax, int64_t nblocks, int dq_blocksize,
                                               const double *run_sums_all, int64_t nblocks_total,
                                               uint8_t *absmax_q, float *absmax2, float *offset,
                                               void *workspace, int64_t workspace_bytes, void *stream);

/* nf4_dequantize -- w~_j = c1' * q[code_j] in binary32 ([MF] "Block-Wise
 * Quantization Mechanics", dequantization equation), with the block constant
 *   c1' = fma(E4M3(absmax_q[b]), absmax2[b/256], *offset)   (one rounding;
 *         READING), or E4M3(absmax_q[b]) * absmax2[b/256] when offset is NULL,
 *   or, when absmax_q is NULL (no double quantization), c1' = absmax2[b]
 *   taken as the fp32 first-level constants absmax[nblocks].
 * NF4_BF16 output is the binary32 value rounded to nearest-even bfloat16 (the
 * compute dtype of [MF] "Forward Pass Computation").
 *   packed     device uint8[n/2]
 *   absmax_q   device uint8[nblocks] or NULL
 *   absmax2    device fp32[ceil(nblocks/256)] (or fp32[nblocks] if absmax_q
 *              is NULL)
 *   offset     device fp32[1] or NULL
 *   n          even, >= 0; blocksize 64; dq_blocksize 256
 *   out        device, n elements of out_dtype (output)
 * One kernel launch. */
NF4_API nf4_status nf4_dequantize(const uint8_t *packed, const uint8_t *absmax_q, const float *absmax2,
                          const float *offset, int64_t n, int blocksize, int dq_blocksize,
                          void *out, nf4_dtype out_dtype, void *stream);

/* Bytes of device workspace nf4_lora_linear_fwd needs for M rows of x and
 * rank r: the low-rank intermediate t (M * round_up(2r, 64) * 2 bytes); 0 for
 * r == 0.  (A library built with NF4_SMALL_M_TC_FROM=9, which sends 9 to 16
 * tokens to the split 16-token tensor-core pipeline, adds that pipeline's
 * scratch for those M: partial tiles and arrival counts, about 3 MiB, after
 * t at a 256-byte boundary.) */
NF4_API int64_t nf4_lora_linear_workspace_size(int64_t M, int r);

/* nf4_lora_linear_fwd -- the frozen-base LoRA linear of [MF] "Forward Pass
 * Computation", Y = X dequant(c1, c2, W) + (alpha/r)(X L1) L2, in weight
 * layout:  y = x W~^T + s (x A^T) B^T,  with W~ the bf16-rounded dequantized
 * weight (dequantized on the fly, never written to memory: [MF] "The
 * dequantization operation does not materialize ..."), bf16 inputs, fp32
 * accumulation, bf16 output.  Internally t = s x A^T is formed first in fp32
 * and kept as a bf16 hi/lo pair (t ~ t_hi + t_lo) in the workspace.
 *   x          device bf16[M, K] row-major
 *   M >= 1, K % 64 == 0, N >= 1
 *   packed, absmax_q, absmax2, offset: the quantized W[N, K] (as for
 *              nf4_dequantize; absmax_q NULL = fp32 first-level constants)
 *   A          device bf16[r, K] or NULL;  B  device bf16[N, r] or NULL
 *   r          0, 16, 32 or 64 (0 or NULL A/B: no low-rank term)
 *   scaling    s = alpha / r
 *   y          device bf16[M, N] (output)
 *   workspace  device scratch, workspace_bytes >=
 *              nf4_lora_linear_workspace_size(M, r); NULL allowed when r == 0.
 *              With r > 0 at least the t part is required (in a library
 *              built with NF4_SMALL_M_TC_FROM=9, a workspace of less than
 *              the full size for 9 <= M <= 16 runs that pipeline unsplit).
 *              Nothing has to be cleared between calls; calls that share a
 *              workspace must be ordered (one stream).
 * M <= 16 runs the streaming warp-MMA decode kernel (one 8-token MMA tile up
 * to M = 8, two above), larger M the tensor-core GEMM pipeline with
 * 256-token tiles; the LoRA pre-step is one extra launch when r > 0. */
NF4_API nf4_status nf4_lora_linear_fwd(const void *x, int64_t M, int64_t K, int64_t N,
                               const uint8_t *packed, const uint8_t *absmax_q,
                               const float *absmax2, const float *offset,
                               const void *A, const void *B, int r, float scaling,
                               void *y, void *workspace, int64_t workspace_bytes, void *stream);

/* Size of the fixed device scratch array behind nf4_lora_linear_fwd_noalloc
 * (4 MiB per GPU that loads the library, held until the process exits). */
#define NF4_NOALLOC_SCRATCH_BYTES (4u * 1024u * 1024u)

/* nf4_lora_linear_fwd_noalloc -- the same operation, arguments and layouts as
 * nf4_lora_linear_fwd, for callers that cannot allocate device memory (a
 * plugin handed only its input and output buffers, a serving loop that must
 * not call cudaMalloc -- which may synchronize the device -- inside a
 * latency-critical step, a framework whose memory is fully reserved by its
 * own pool).  There is no workspace argument: the low-rank intermediate lives
 * in a fixed device array inside the library.  The pages have no counterpart
 * to this entry point; it is an interface convenience only.
 *   Limit: the intermediate t, M * round_up(2r, 64) * 2 bytes, must not
 *          exceed NF4_NOALLOC_SCRATCH_BYTES (M <= 16384 for r = 64, M <= 32768
 *          for r <= 32); larger sizes return NF4_ERR_UNSUPPORTED before any
 *          work.  (In a library built with NF4_SMALL_M_TC_FROM=9 the array
 *          also holds, for 9 to 16 tokens, the split pipeline's
 *          scratch: nf4_lora_linear_workspace_size(M, r) <= 4 MiB there.)
 *   The first call on a device looks up the array's device address (with
 *   that device current); make that first call before any stream capture.
 *   The address is cached for the life of the process's context on that
 *   device: after cudaDeviceReset (or anything else that destroys the
 *   primary context) this entry point must not be called again in the
 *   same process.
 *   All calls on a device share the array: calls whose kernels may overlap on
 *   the GPU (unordered streams) race and give undefined results.  Nothing has
 *   to be cleared between calls.
 *   Never calls cudaMalloc, cudaFree or any allocating routine. */
NF4_API nf4_status nf4_lora_linear_fwd_noalloc(const void *x, int64_t M, int64_t K, int64_t N,
                                               const uint8_t *packed, const uint8_t *absmax_q,
                                               const float *absmax2, const float *offset,
                                               const void *A, const void *B, int r, float scaling,
                                               void *y, void *stream);

/* nf4_device_status -- synchronize `stream`, then read and clear the
 * library's device error word on the current device.  Returns
 * NF4_ERR_TIMEOUT if a bounded wait in a kernel expired since the last call,
 * NF4_ERR_CUDA on a CUDA error, NF4_OK otherwise. */
NF4_API nf4_status nf4_device_status(void *stream);

/* nf4_lora_linear_bwd_workspace_size -- bytes of device workspace that
 * nf4_lora_linear_bwd needs for these sizes (0 when r = 0). */
NF4_API int64_t nf4_lora_linear_bwd_workspace_size(int64_t M, int64_t N, int64_t K, int r);

/* nf4_lora_linear_bwd -- backward pass of nf4_lora_linear_fwd ("QLoRA:
 * Mathematical Foundations ...", section "Gradient Computation": gradients go
 * to the adapter only; the activation gradient flows through both paths).  In
 * the layout W[N, K], A[r, K], B[N, r], with g = dL/dy bf16 [M, N]:
 *   dx = g W~ + s (g B) A            bf16 [M, K] (W~ = bf16 dequantized W,
 *                                    exactly nf4_dequantize's output)
 *   dA = s (g B)^T x                 fp32 [r, K]
 *   dB = s g^T (x A^T)               fp32 [N, r]
 * bf16 operands, fp32 accumulation.  Any of dx, dA, dB may be NULL (not
 * computed); x is needed only for dA and dB; A, B NULL or r = 0 drop the
 * adapter (then dA, dB must be NULL).
 *   g, x, A, B, packed, absmax_q, absmax2, offset: as for nf4_lora_linear_fwd
 *       (device pointers, 16-byte aligned, caller-owned).
 *   N % 8 == 0 (rows of g are read by TMA), K % 64 == 0, r in {0,16,32,64}.
 *   workspace: >= nf4_lora_linear_bwd_workspace_size(M, N, K, r) bytes of
 *       device memory, 256-byte aligned (scratch: s g B as a bf16 hi/lo pair,
 *       B^T and A^T).
 * Errors: NF4_ERR_INVALID, NF4_ERR_UNSUPPORTED (r or shapes outside the
 * above), NF4_ERR_CUDA.  Asynchronous on stream; NF4_ERR_TIMEOUT (a bounded
 * wait expired) is reported by nf4_device_status. */
NF4_API nf4_status nf4_lora_linear_bwd(const void *g, const void *x, int64_t M, int64_t K, int64_t N,
                                       const uint8_t *packed, const uint8_t *absmax_q, const float *absmax2,
                                       const float *offset, const void *A, const void *B, int r, float scaling,
                                       void *dx, float *dA, float *dB, void *workspace, int64_t workspace_bytes,
                                       void *stream);

/* nf4_merge_requantize -- merge the LoRA adapter into the quantized base and
 * quantize the result again ("QLoRA in Production ...", section "Step 4:
 * Merging and Inference"; "QLoRA: quantising the part you are not training",
 * section "What it costs", item 3: a merge into the quantized base must be
 * requantized).  READING of the arithmetic (the pages give none), in binary32:
 *   w~[n, k] = RN(q[code] * c1')                      (as nf4_dequantize, fp32)
 *   d[n, k]  = chain d <- fma(B[n, j], A[j, k], d), j = 0 .. r-1, from +0
 *   W'[n, k] = fma(scaling, d[n, k], w~[n, k])
 * then blockwise NF4 of W' (as nf4_quantize on an fp32 tensor).
 *   packed, absmax_q, absmax2, offset: the quantized W[N, K], as for
 *       nf4_dequantize (absmax_q NULL: absmax2 holds fp32 constants;
 *       offset NULL: no centring).  K % 64 == 0.
 *   A: bf16 [r, K], B: bf16 [N, r] (device), 0 <= r <= 64 (r = 0 or NULL A/B:
 *       no adapter, W' = w~).
 *   packed_out: uint8 [N K / 2], absmax_out: fp32 [N K / 64] (device),
 *       caller-owned; packed_out may alias packed, absmax_out may alias
 *       absmax2 when absmax_q is NULL.  Double-quantize absmax_out with
 *       nf4_double_quantize to return to the stored format.
 * Errors: NF4_ERR_INVALID (null or misaligned pointers, N < 1, K not a
 * positive multiple of 64, offset without absmax_q), NF4_ERR_UNSUPPORTED
 * (r > 64), NF4_ERR_CUDA on a launch error.  Asynchronous on stream. */
NF4_API nf4_status nf4_merge_requantize(const uint8_t *packed, const uint8_t *absmax_q, const float *absmax2,
                                        const float *offset, int64_t N, int64_t K, const void *A, const void *B,
                                        int r, float scaling, uint8_t *packed_out, float *absmax_out, void *stream);

/* nf4_selftest_wait_timeout -- failure-detection check (no counterpart on
 * the pages).  Launches on `stream` one thread that waits on a shared-memory
 * mbarrier nothing arrives on; after limit_ns nanoseconds of %globaltimer
 * (1 <= limit_ns <= 1e9) it raises the device error word and returns, as the
 * fused kernels do when one of their bounded waits expires.  The GPU is
 * neither faulted nor hung and the context stays usable.  Returns NF4_OK once
 * launched (NF4_ERR_INVALID for a limit out of range, NF4_ERR_CUDA on a launch
 * error); the following nf4_device_status() returns NF4_ERR_TIMEOUT and
 * clears the word. */
NF4_API nf4_status nf4_selftest_wait_timeout(int64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* NF4_H_ */
