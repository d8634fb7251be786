/* decode_split.h -- how the decode kernel (decode.cu) shares out its work,
 * in plain C++ so that the kernel and a CPU test harness compile the same
 * code.
 *
 * Row tiles of 16 weight rows; CTA c of G takes the contiguous tiles
 * [c T / G, (c + 1) T / G) of the T tiles.  A unit is (tile, slice): 16 rows
 * x 256 / nt columns, nt = the number of 8-token MMA tiles (1 up to 8
 * tokens, 2 up to 16), so a row has S = ceil(K / (256 / nt)) slices.
 *   - S <= 16: warp w takes slice w % S of the tiles w / S, w / S + tps,
 *     ... (tps = 16 / S tiles per round of the 16 warps); its partial tiles
 *     go to slot = slice.
 *   - S > 16: warp w takes slices w, w + 16, ... of every tile; inside a
 *     chunk of tiles it runs them slice-major (every tile of the chunk at
 *     slice w, then at w + 16, ...), so that its x fragments are loaded once
 *     per slice and chunk; its partial tiles go to slot = w, written at the
 *     first slice (w < 16) and accumulated at the later ones in slice order.
 * The partial tiles of a chunk (nslot slots of 128 nt floats per tile) live
 * in two shared-memory regions: the first low_tiles tiles below the decode
 * kernel's level-pair table, the rest after its rings.  A chunk is a
 * multiple of tps tiles unless it covers all of a CTA's tiles. */
#ifndef NF4_DECODE_SPLIT_H_
#define NF4_DECODE_SPLIT_H_

#include <stdint.h>

#if defined(__CUDACC__)
#define NF4_DS_FN __host__ __device__ __forceinline__
#else
#define NF4_DS_FN inline
#endif

namespace nf4 {

constexpr int kDWarps = 16;
constexpr int kDRing = 3;           // unit slots per warp
constexpr int kDSmem = 227 * 1024;  // dynamic shared memory per CTA: all of it
// Shared-window offsets: the pair table at 64 KB (so that a code byte
// permuted into bits 8..15 addresses its entry), the rings at 128 KB, the
// low partials from the dynamic base (below 1 KB) up to the table.
constexpr uint32_t kDTableAt = 0x10000, kDRingAt = 0x20000;
constexpr uint32_t kDPartRoom = kDTableAt - 1024;

// Bytes of the 16 warps' rings: kDRing units of 16 rows x 128 / nt bytes each.
NF4_DS_FN constexpr int64_t decode_ring_bytes(int nt) { return (int64_t)kDWarps * kDRing * 16 * (128 / nt); }
// 64-blocks of a row in a unit, and the unit's slices per row.
NF4_DS_FN constexpr int decode_blocks_per_unit(int nt) { return 4 / nt; }
NF4_DS_FN constexpr int64_t decode_slices(int64_t K, int nt) {
    return (K / 64 + decode_blocks_per_unit(nt) - 1) / decode_blocks_per_unit(nt);
}

// Work of one CTA: tiles [t0, t0 + my_tiles) in chunks of `chunk` tiles, S
// slices per row.
struct DWork {
    int64_t t0;
    int my_tiles, S, tps, nslot, chunk;
    int tw, s_w;  // S <= 16: first tile and slice of this warp
    bool active;  // S <= 16: the warp has a slice

    // n_tiles * ctas < 2^32 (checked by the host): 32-bit divisions
    NF4_DS_FN void init(uint32_t n_tiles, int64_t K, int nt, int warp, int chunk_tiles, uint32_t cta,
                        uint32_t ctas) {
        const uint32_t b0 = cta * n_tiles / ctas, b1 = (cta + 1) * n_tiles / ctas;
        t0 = b0;
        my_tiles = (int)(b1 - b0);
        S = (int)decode_slices(K, nt);
        chunk = chunk_tiles;
        tps = S <= kDWarps ? kDWarps / S : 1;
        nslot = S < kDWarps ? S : kDWarps;
        tw = S <= kDWarps ? warp / S : 0;
        s_w = S <= kDWarps ? warp % S : warp;
        active = S > kDWarps || warp < tps * S;
    }
};

// Position in a warp's unit sequence: tile j (in the CTA), slice s; cb =
// first tile of the current chunk.
struct DCursor {
    int j, s, cb;
    NF4_DS_FN void start(const DWork &wk) {
        j = wk.active ? wk.tw : wk.my_tiles;
        s = wk.s_w;
        cb = 0;
    }
    NF4_DS_FN void step(const DWork &wk, int warp) {
        if (wk.S <= kDWarps) {
            j += wk.tps;
            return;
        }
        const int ce = cb + wk.chunk < wk.my_tiles ? cb + wk.chunk : wk.my_tiles;
        if (++j < ce) return;
        if ((s += kDWarps) < wk.S) {
            j = cb;
            return;
        }
        s = warp;  // the next chunk, which starts at j == ce
        cb = ce;
    }
    NF4_DS_FN bool valid(const DWork &wk) const { return j < wk.my_tiles; }
    // partial-tile slot of the current unit
    NF4_DS_FN int slot(const DWork &wk, int warp) const { return wk.S <= kDWarps ? s : warp; }
};

// Host side: the grid (one CTA per SM, at most one per tile) and the tiles
// of a chunk.  Returns false when the call cannot be split (32-bit work
// split, or not one tile's partials fit).
struct DChunk {
    int grid, chunk, low_tiles;
};
NF4_DS_FN bool decode_chunk(int64_t N, int64_t K, int nt, int num_sms, DChunk *out) {
    const int64_t n_tiles = (N + 15) / 16;
    const int grid = (int)(n_tiles < num_sms ? n_tiles : num_sms);
    if (grid < 1 || n_tiles * (grid + 1) >= ((int64_t)1 << 32)) return false;
    const int64_t S = decode_slices(K, nt);
    const int64_t nslot = S < kDWarps ? S : kDWarps, tps = S <= kDWarps ? kDWarps / S : 1;
    const int64_t max_tiles = (n_tiles + grid - 1) / grid;
    const int64_t tile_bytes = nslot * 128 * nt * 4;
    const int64_t low = kDPartRoom / tile_bytes;
    const int64_t high = ((int64_t)kDSmem - (kDRingAt + decode_ring_bytes(nt))) / tile_bytes;
    int64_t chunk = low + high;
    if (chunk >= max_tiles) chunk = max_tiles;
    else chunk -= chunk % tps;
    if (chunk < 1) return false;
    out->grid = grid;
    out->chunk = (int)chunk;
    out->low_tiles = (int)(low < chunk ? low : chunk);
    return true;
}

}  // namespace nf4

#endif /* NF4_DECODE_SPLIT_H_ */
