// Test helper: runs the decode kernel's work split for every CTA and warp of
// a call on the CPU, with the functions of the kernel's own header
// (csrc/decode_split.h), and checks what the kernel relies on.
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>

#include <vector>

#include "decode_split.h"

using namespace nf4;

namespace {

int fail(char *msg, int len, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(msg, (size_t)len, fmt, ap);
    va_end(ap);
    return 1;
}

}  // namespace

extern "C" int ds_chunk(int64_t N, int64_t K, int nt, int num_sms, int *grid, int *chunk, int *low_tiles) {
    DChunk ch;
    if (!decode_chunk(N, K, nt, num_sms, &ch)) return 0;
    *grid = ch.grid;
    *chunk = ch.chunk;
    *low_tiles = ch.low_tiles;
    return 1;
}

// 0 when every check holds, else 1 with the first failure in msg.
extern "C" int ds_check(int64_t N, int64_t K, int nt, int num_sms, char *msg, int msglen) {
    DChunk ch;
    if (!decode_chunk(N, K, nt, num_sms, &ch)) return fail(msg, msglen, "no split");
    const int64_t n_tiles = (N + 15) / 16;
    const int S = (int)decode_slices(K, nt);
    const int nslot = S < kDWarps ? S : kDWarps, tps = S <= kDWarps ? kDWarps / S : 1;
    const int64_t tile_bytes = (int64_t)nslot * 128 * nt * 4;
    const int64_t ring_end = kDRingAt + decode_ring_bytes(nt);
    // shared-memory regions: rings inside the allocation, low partials below
    // the table, high partials after the rings
    if (ring_end > kDSmem) return fail(msg, msglen, "rings end at %lld", (long long)ring_end);
    if (ch.low_tiles < 0 || ch.low_tiles > ch.chunk || ch.low_tiles * tile_bytes > kDPartRoom)
        return fail(msg, msglen, "low region: %d tiles of %lld bytes", ch.low_tiles, (long long)tile_bytes);
    if (ring_end + (ch.chunk - ch.low_tiles) * tile_bytes > kDSmem)
        return fail(msg, msglen, "high region: %d tiles", ch.chunk - ch.low_tiles);
    if (ch.grid < 1 || ch.grid > num_sms || ch.grid > n_tiles) return fail(msg, msglen, "grid %d", ch.grid);

    int64_t covered = 0;
    for (int cta = 0; cta < ch.grid; ++cta) {
        DWork w0;
        w0.init((uint32_t)n_tiles, K, nt, 0, ch.chunk, (uint32_t)cta, (uint32_t)ch.grid);
        if (w0.t0 != covered) return fail(msg, msglen, "cta %d starts at tile %lld", cta, (long long)w0.t0);
        if (w0.my_tiles < 1) return fail(msg, msglen, "cta %d has no tile", cta);
        covered += w0.my_tiles;
        if (ch.chunk < w0.my_tiles && ch.chunk % tps != 0)
            return fail(msg, msglen, "chunk %d not a multiple of %d", ch.chunk, tps);
        const int my = w0.my_tiles;
        std::vector<int> seen((size_t)my * S, 0);
        std::vector<int> last_s((size_t)my * kDWarps, -1);  // per (tile, slot): last slice added
        for (int warp = 0; warp < kDWarps; ++warp) {
            DWork wk;
            wk.init((uint32_t)n_tiles, K, nt, warp, ch.chunk, (uint32_t)cta, (uint32_t)ch.grid);
            DCursor c;
            c.start(wk);
            int x_slice = -1, x_loads = 0, nchunks = 0;
            int64_t units = 0;
            for (int c0 = 0; c0 < my; c0 += ch.chunk) {
                ++nchunks;
                const int c1 = my - c0 < ch.chunk ? my : c0 + ch.chunk;
                for (; c.valid(wk) && c.j < c1; c.step(wk, warp)) {
                    if (++units > (int64_t)my * S)
                        return fail(msg, msglen, "cta %d warp %d: more units than the tiles hold", cta, warp);
                    const int j = c.j, s = c.s, sl = c.slot(wk, warp);
                    if (j < c0) return fail(msg, msglen, "cta %d warp %d: tile %d before its chunk", cta, warp, j);
                    if (s < 0 || s >= S) return fail(msg, msglen, "slice %d of %d", s, S);
                    if (sl < 0 || sl >= nslot) return fail(msg, msglen, "slot %d of %d", sl, nslot);
                    if (S <= kDWarps) {
                        if (s != warp % S || sl != s || (j - warp / S) % tps != 0)
                            return fail(msg, msglen, "warp %d: unit (%d, %d) outside its slice", warp, j, s);
                    } else if (sl != warp || s % kDWarps != warp) {
                        return fail(msg, msglen, "warp %d: slice %d, slot %d", warp, s, sl);
                    }
                    ++seen[(size_t)j * S + s];
                    // a slot's partial tile is written by its first unit
                    // (s < 16) and accumulated in increasing slice order
                    int &ls = last_s[(size_t)j * kDWarps + sl];
                    if (ls < 0 ? s >= kDWarps : (s < kDWarps || s <= ls))
                        return fail(msg, msglen, "tile %d slot %d: slice %d after %d", j, sl, s, ls);
                    ls = s;
                    if (s != x_slice) {
                        x_slice = s;
                        ++x_loads;
                    }
                }
            }
            if (c.valid(wk)) return fail(msg, msglen, "cta %d warp %d: units left after the chunks", cta, warp);
            const int my_slices = S <= kDWarps ? 1 : (S - warp + kDWarps - 1) / kDWarps;
            if (wk.active && x_loads > nchunks * my_slices)
                return fail(msg, msglen, "warp %d loads x %d times (%d chunks, %d slices)", warp, x_loads, nchunks,
                            my_slices);
        }
        for (int64_t i = 0; i < (int64_t)my * S; ++i)
            if (seen[(size_t)i] != 1)
                return fail(msg, msglen, "cta %d: unit (%lld, %lld) run %d times", cta, (long long)(i / S),
                            (long long)(i % S), seen[(size_t)i]);
    }
    if (covered != n_tiles) return fail(msg, msglen, "tiles covered %lld of %lld", (long long)covered, (long long)n_tiles);
    return 0;
}
