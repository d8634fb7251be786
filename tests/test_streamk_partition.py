"""Host-side check of the work partition that the split 16-token pipeline
(decode calls of 9 to 16 tokens in a library built with
NF4_SMALL_M_TC_FROM=9) relies on: the partition functions are
compiled from the kernel's own header (csrc/streamk.h) with gcc and checked
by exhaustion over many shapes:

  - CTA c of G runs the global steps [c T / G, (c + 1) T / G) of the
    T = tiles x kt_total steps (tile-major); every step is run exactly once;
  - with more CTAs than tiles a range covers the end of one tile and the
    start of the next at most (two segments, two accumulators);
  - the owner of step s is (s G + G - 1) / T, so a tile's contributors are
    the CTAs from the owner of its first step to the owner of its last, and
    a contributor's segment is 0 when its range starts in that tile, else 1;
  - the arrival count that completes a tile equals its number of
    contributors (one arrival per contributing segment).

The GPU tests check the kernel itself against the oracle; this one pins the
arithmetic of the scheme on shapes the GPU tests cannot all reach."""
import ctypes
import os
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(os.path.dirname(HERE), "qlora_nf4_quantize_b200", "csrc")


@pytest.fixture(scope="module")
def sk(tmp_path_factory):
    so = str(tmp_path_factory.mktemp("sk") / "streamk_harness.so")
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-I", CSRC, os.path.join(HERE, "helpers", "streamk_harness.c"),
                    "-o", so], check=True)
    L = ctypes.CDLL(so)
    i64 = ctypes.c_int64
    L.sk_begin.restype = i64
    L.sk_begin.argtypes = [i64, i64, i64]
    L.sk_owner.restype = i64
    L.sk_owner.argtypes = [i64, i64, i64]
    L.sk_segment.restype = ctypes.c_int
    L.sk_segment.argtypes = [i64, i64, i64, i64, i64]
    return L


def check_shape(sk, ntiles, kt_total, ctas):
    total = ntiles * kt_total
    lo = [sk.sk_begin(c, total, ctas) for c in range(ctas + 1)]
    assert lo[0] == 0 and lo[ctas] == total
    runs = [0] * total
    contributors = {t: [] for t in range(ntiles)}
    for c in range(ctas):
        g_lo, g_hi = lo[c], lo[c + 1]
        assert g_hi > g_lo, "every CTA gets at least one step"
        tile0, kt_first = divmod(g_lo, kt_total)
        steps, i_next = g_hi - g_lo, kt_total - kt_first
        nseg = 2 if steps > i_next else 1
        for i in range(steps):
            seg = 1 if i >= i_next else 0
            kt = i - i_next if seg else kt_first + i
            assert 0 <= kt < kt_total
            s = (tile0 + seg) * kt_total + kt
            assert s == g_lo + i
            runs[s] += 1
        for seg in range(nseg):
            contributors[tile0 + seg].append((c, seg))
        assert steps - i_next < kt_total, "at most two segments"
    assert all(r == 1 for r in runs)
    for t in range(ntiles):
        c0, c1 = sk.sk_owner(t * kt_total, total, ctas), sk.sk_owner(t * kt_total + kt_total - 1, total, ctas)
        listed = [(c, sk.sk_segment(c, t, kt_total, total, ctas)) for c in range(c0, c1 + 1)]
        assert listed == contributors[t]
        assert len(listed) == c1 - c0 + 1  # the count that completes the tile


@pytest.mark.parametrize("ntiles,kt_total,ctas", [(86, 65, 148), (86, 65, 140), (1, 17, 2), (19, 9, 21),
                                                  (19, 10, 23), (8, 129, 64), (147, 2, 148)])
def test_partition_of_measured_and_tested_shapes(sk, ntiles, kt_total, ctas):
    check_shape(sk, ntiles, kt_total, ctas)


def test_partition_exhaustive_small(sk):
    for ntiles in range(1, 40):
        for kt_total in (1, 2, 3, 8, 9, 17, 65, 66):
            total = ntiles * kt_total
            for ctas in range(ntiles + 1, min(total, 160) + 1, 3):
                check_shape(sk, ntiles, kt_total, ctas)
