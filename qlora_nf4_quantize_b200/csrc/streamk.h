/* streamk.h -- the work partition of the split 16-token decode pipeline
 * (gemm_tc.cu, stream-K; taken for 9 to 16 tokens in a library built with
 * NF4_SMALL_M_TC_FROM=9), in plain C so that the kernel and a CPU test
 * harness compile the same functions.
 *
 * The T = tiles x kt_total (weight tile, k-step) pairs are taken tile after
 * tile; CTA c of G runs the contiguous range [c T / G, (c + 1) T / G).  With
 * more CTAs than tiles a range covers the end of one tile and the start of
 * the next at most (its segments 0 and 1).  The CTAs that contribute to a
 * tile are those from the owner of its first step to the owner of its last;
 * a contributor's segment for the tile is 0 when its range starts in that
 * tile, else 1. */
#ifndef NF4_STREAMK_H_
#define NF4_STREAMK_H_

#include <stdint.h>

#if defined(__CUDACC__)
#define NF4_SK_FN __host__ __device__ __forceinline__
#else
#define NF4_SK_FN static inline
#endif

/* First global step of CTA c's range (c = G gives T, the end). */
NF4_SK_FN int64_t nf4_sk_begin(int64_t c, int64_t total, int64_t ctas) { return c * total / ctas; }

/* CTA whose range holds global step s: the largest c with c T / G <= s. */
NF4_SK_FN int64_t nf4_sk_owner(int64_t s, int64_t total, int64_t ctas) { return (s * ctas + ctas - 1) / total; }

/* Segment (0 or 1) in which contributor c adds to tile `tile`. */
NF4_SK_FN int nf4_sk_segment(int64_t c, int64_t tile, int64_t kt_total, int64_t total, int64_t ctas) {
    return nf4_sk_begin(c, total, ctas) / kt_total == tile ? 0 : 1;
}

#endif /* NF4_STREAMK_H_ */
