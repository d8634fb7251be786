/* Test helper: exhaustive sweep over every binary32 value in [-1, 1].
 * For each x it compares code_of(x) (the function under test, passed as a
 * pointer) with the threshold count #{i : x > t[i]} for 15 thresholds given
 * by the caller.  Returns the number of mismatches; *first receives the bit
 * pattern of the first mismatch found. */
#include <stdint.h>
#include <string.h>

typedef int (*code_fn)(float);

int64_t sweep_all(code_fn code_of, const float *t, uint32_t *first) {
    int64_t bad = 0;
    uint32_t firstbad = 0xFFFFFFFFu;
    const uint32_t one = 0x3F800000u; /* bits of 1.0f */
#pragma omp parallel for schedule(static, 1 << 20) reduction(+ : bad)
    for (int64_t u = 0; u <= (int64_t)one; ++u) {
        for (int s = 0; s < 2; ++s) {
            uint32_t bits = (uint32_t)u | (s ? 0x80000000u : 0u);
            float x;
            memcpy(&x, &bits, 4);
            int c = 0;
            for (int i = 0; i < 15; ++i) c += (x > t[i]);
            if (code_of(x) != c) {
                ++bad;
#pragma omp critical
                if (bits < firstbad) firstbad = bits;
            }
        }
    }
    *first = firstbad;
    return bad;
}
