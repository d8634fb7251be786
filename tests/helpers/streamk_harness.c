/* Test helper: exports the split decode pipeline's partition functions,
 * compiled from the very header the kernel includes (csrc/streamk.h). */
#include <stdint.h>

#include "streamk.h"

int64_t sk_begin(int64_t c, int64_t total, int64_t ctas) { return nf4_sk_begin(c, total, ctas); }
int64_t sk_owner(int64_t s, int64_t total, int64_t ctas) { return nf4_sk_owner(s, total, ctas); }
int sk_segment(int64_t c, int64_t tile, int64_t kt_total, int64_t total, int64_t ctas) {
    return nf4_sk_segment(c, tile, kt_total, total, ctas);
}
