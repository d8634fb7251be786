"""Host-side check of how the decode kernel (csrc/decode.cu) shares out its
work: the split is compiled from the kernel's own header
(csrc/decode_split.h) with g++ and run for every CTA and warp of a call, over
many shapes and both token-tile counts:

  - the CTAs take contiguous, disjoint tile ranges that cover every row tile;
  - every (tile, slice) unit of a CTA runs exactly once, inside the chunk
    it belongs to, and no warp has units left after the last chunk;
  - with at most 16 slices a warp keeps one slice (its x fragments stay in
    registers) and its partial tiles go to that slice's slot; with more, a
    warp takes slices w, w + 16, ... into slot w;
  - a slot's partial tile is first written (slice < 16) and then only
    accumulated, in increasing slice order, so the sum does not depend on
    timing;
  - with more than 16 slices a warp loads x at most once per slice and chunk;
  - the partial tiles of a chunk fit the two shared-memory regions (below
    the level-pair table, after the rings), and a chunk is a multiple of the
    tiles one round of the warps covers unless it holds all of a CTA's tiles.

The GPU tests check the kernel against the oracle on shapes that reach each
way of splitting; this one pins the split itself on many more."""
import ctypes
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "qlora_nf4_quantize_b200", "csrc")


@pytest.fixture(scope="module")
def ds(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("ds") / "decode_split_harness.so")
    subprocess.run(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-I", CSRC,
                    os.path.join(HERE, "helpers", "decode_split_harness.cpp"), "-o", so], check=True)
    L = ctypes.CDLL(so)
    i64, i32 = ctypes.c_int64, ctypes.c_int
    L.ds_check.restype = i32
    L.ds_check.argtypes = [i64, i64, i32, i32, ctypes.c_char_p, i32]
    L.ds_chunk.restype = i32
    L.ds_chunk.argtypes = [i64, i64, i32, i32] + [ctypes.POINTER(i32)] * 3
    return L


def check(ds, N, K, nt, sms):
    buf = ctypes.create_string_buffer(256)
    rc = ds.ds_check(N, K, nt, sms, buf, 256)
    assert rc == 0, f"N={N} K={K} nt={nt} sms={sms}: {buf.value.decode()}"


def chunk(ds, N, K, nt, sms):
    g, c, lo = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    assert ds.ds_chunk(N, K, nt, sms, ctypes.byref(g), ctypes.byref(c), ctypes.byref(lo)) == 1
    return g.value, c.value, lo.value


@pytest.mark.parametrize("nt", [1, 2])
def test_split_invariants(ds, nt):
    for K in (64, 128, 192, 256, 320, 1024, 1344, 2048, 4096, 5120, 8192, 11008, 14336):
        for N in (1, 8, 16, 17, 40, 136, 264, 520, 1024, 4000, 4096, 11008, 14336):
            for sms in (1, 5, 140, 148):
                check(ds, N, K, nt, sms)


@pytest.mark.parametrize("nt", [1, 2])
def test_split_many_tiles_per_cta(ds, nt):
    """More tiles per CTA than one chunk's partials hold (several chunks)."""
    for K in (64, 512, 4096, 14336):
        for N in (33024, 65536, 100000):
            for sms in (16, 140):
                check(ds, N, K, nt, sms)


def test_chunks_of_the_decode_workload(ds):
    """W 11008 x 4096 on 140 CTAs (an adapter leaves 8 SMs to the
    down-projection): 688 tiles, 4-5 per CTA.  One token tile: 16 slices of
    256 columns, 8 KB of partials per tile, all 5 tiles below the table.
    Two token tiles: 32 slices of 128 columns, 16 KB per tile, 3 below the
    table and 2 after the 48 KB of rings."""
    assert chunk(ds, 11008, 4096, 1, 140) == (140, 5, 5)
    assert chunk(ds, 11008, 4096, 2, 140) == (140, 5, 3)
    # one CTA with every tile: chunks of 7 (one tile) and 6 (two tiles)
    assert chunk(ds, 11008, 4096, 1, 1) == (1, 7, 7)
    assert chunk(ds, 11008, 4096, 2, 1) == (1, 6, 3)
