"""Pins of the oracle's blockwise NF4 quantization and dequantization.

The definition ("QLoRA: Mathematical Foundations ...", section "Block-Wise
Quantization Mechanics"): c1 = max |w| per contiguous block of 64, code =
arg-min_i |w / c1 - q_i|, w~ = c1 * q[code].  Pins: exact rational arg-min on
samples, an exhaustive sweep of every binary32 in [-1, 1] against the
threshold form, brute force on tiny hand-made tensors, the round-trip error
bound, and the qualitative NF4-beats-uniform-int4 claim of "QLoRA in
Production ..." (section "1. 4-bit NormalFloat").
"""
import ctypes
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest

import nf4_workloads as wl

HERE = os.path.dirname(os.path.abspath(__file__))


def exact_levels(oracle_mod):
    return [Fraction(float(v)) for v in oracle_mod.codebook()]


def exact_argmin(x, levels):
    """Brute-force nearest level in exact rational arithmetic; first minimum."""
    xf = Fraction(float(x))
    d = [abs(xf - q) for q in levels]
    return d.index(min(d))


def thresholds_rd(levels):
    """t_i = largest binary32 <= (q_i + q_{i+1}) / 2, computed exactly."""
    ts = []
    for a, b in zip(levels[:-1], levels[1:]):
        m = (a + b) / 2
        t = np.float32(float(m))  # nearest; step down if above m
        if Fraction(float(t)) > m:
            t = np.nextafter(t, np.float32(-2.0))
        ts.append(t)
    return np.array(ts, np.float32)


def test_levels_map_to_themselves(oracle_mod):
    for i, q in enumerate(oracle_mod.codebook()):
        assert oracle_mod.code_of(q) == i


def test_midpoint_ties_go_to_lower_index(oracle_mod):
    L = exact_levels(oracle_mod)
    n_repr = 0
    for i in range(15):
        m = (L[i] + L[i + 1]) / 2
        mf = np.float32(float(m))
        if Fraction(float(mf)) == m:  # midpoint exactly representable: a tie
            n_repr += 1
            assert oracle_mod.code_of(mf) == i
            assert oracle_mod.code_of(np.nextafter(mf, np.float32(2))) == i + 1
            assert oracle_mod.code_of(np.nextafter(mf, np.float32(-2))) == i
    assert n_repr >= 1  # the pages' table does contain reachable ties


def test_code_of_matches_exact_argmin_on_samples(oracle_mod):
    L = exact_levels(oracle_mod)
    rng = np.random.default_rng(0)
    xs = np.concatenate([
        rng.uniform(-1, 1, 3000).astype(np.float32),
        (rng.standard_normal(1000) * 0.3).clip(-1, 1).astype(np.float32),
        np.array([0.0, -0.0, 1e-40, -1e-40, 1.0, -1.0], np.float32),
    ])
    # values a few ulps around every midpoint
    for i in range(15):
        m = np.float32(float((L[i] + L[i + 1]) / 2))
        v = m
        for _ in range(4):
            v = np.nextafter(v, np.float32(-2))
        for _ in range(9):
            xs = np.append(xs, v)
            v = np.nextafter(v, np.float32(2))
    got = oracle_mod.code_of_array(xs)
    want = np.array([exact_argmin(x, L) for x in xs])
    assert np.array_equal(got, want)


def test_code_of_exhaustive_against_threshold_form(oracle_mod, tmp_path):
    """Every binary32 in [-1, 1] (about 2.1e9 values)."""
    so = tmp_path / "code_sweep.so"
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", os.path.join(HERE, "helpers", "code_sweep.c"),
                    "-o", str(so)], check=True)
    helper = ctypes.CDLL(str(so))
    helper.sweep_all.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    helper.sweep_all.restype = ctypes.c_int64
    t = thresholds_rd(exact_levels(oracle_mod))
    first = ctypes.c_uint32(0)
    fn = ctypes.cast(oracle_mod.lib().nf4o_code_of, ctypes.c_void_p)
    bad = helper.sweep_all(fn, t.ctypes.data_as(ctypes.c_void_p), ctypes.byref(first))
    assert bad == 0, f"first mismatch at bits {first.value:#010x}"


def brute_quantize(w32, bs, levels):
    """Tiny-tensor brute force straight from the definition."""
    n = w32.size
    codes, absmax = [], []
    for lo in range(0, n, bs):
        blk = w32[lo:lo + bs]
        c1 = max(abs(float(v)) for v in blk)
        absmax.append(c1)
        for v in blk:
            if c1 == 0:
                codes.append(7)
            else:
                x = np.float32(np.float32(v) / np.float32(c1))  # IEEE binary32 quotient
                codes.append(exact_argmin(x, levels))
    packed = [(codes[2 * j] << 4) | codes[2 * j + 1] for j in range(n // 2)]
    return np.array(packed, np.uint8), np.array(absmax, np.float32)


def test_quantize_hand_cases_bruteforce(oracle_mod):
    L = exact_levels(oracle_mod)
    rng = np.random.default_rng(1)
    w = (rng.standard_normal(64 * 5 + 18) * 0.02).astype(np.float32)
    w[64:128] = 0.0                       # all-zero block
    w[130] = -0.0
    w[200] = 0.4                          # outlier in block 3
    w[256:320] = -w[256:320]              # negative block
    w[5] = -0.0
    packed, absmax = oracle_mod.quantize(w, 64)
    bp, ba = brute_quantize(w, 64, L)
    assert np.array_equal(absmax, ba)
    assert np.array_equal(packed, bp)
    assert absmax[1] == 0 and np.all(packed[32:64] == 0x77)


def test_quantize_bf16_equals_widened_f32(oracle_mod):
    import torch
    wt = wl.weight((64, 128), 0.02, 7, "bf16")
    bits = wt.view(torch.int16).numpy().view(np.uint16).ravel()
    p1, a1 = oracle_mod.quantize(bits)
    p2, a2 = oracle_mod.quantize(wt.float().numpy().ravel())
    assert np.array_equal(p1, p2) and np.array_equal(a1, a2)


def level_gap_bound(levels_f64, code):
    lo = levels_f64[code] - levels_f64[code - 1] if code > 0 else 0.0
    hi = levels_f64[code + 1] - levels_f64[code] if code < 15 else 0.0
    return max(lo, hi)


def test_round_trip_error_bound_no_dq(oracle_mod):
    """|w - w~| <= c1 * (g/2 + 2^-22), g the larger gap beside the chosen level."""
    w = wl.weight_case(wl.TINY).numpy().ravel()
    packed, absmax = oracle_mod.quantize(w)
    wt = oracle_mod.dequantize(packed, None, absmax, None, w.size)
    q = oracle_mod.codebook().astype(np.float64)
    codes = np.empty(w.size, np.int64)
    codes[0::2] = packed >> 4
    codes[1::2] = packed & 15
    c1 = np.repeat(absmax.astype(np.float64), 64)[: w.size]
    bound = np.array([level_gap_bound(q, c) for c in codes]) * 0.5 * c1 + c1 * 2.0 ** -22
    err = np.abs(w.astype(np.float64) - wt.astype(np.float64))
    assert np.all(err <= bound)
    # and the reconstruction is exactly c1 * q[code] in binary32
    assert np.array_equal(wt, c1.astype(np.float32) * q[codes].astype(np.float32))


def test_dequantize_bf16_is_rne_of_f32(oracle_mod):
    import torch
    w = wl.weight_case(wl.TINY).numpy().ravel()
    packed, absmax = oracle_mod.quantize(w)
    f = oracle_mod.dequantize(packed, None, absmax, None, w.size, "f32")
    b = oracle_mod.dequantize(packed, None, absmax, None, w.size, "bf16")
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(b, ref)


def test_nf4_beats_uniform_int4_on_gaussian(oracle_mod):
    """Qualitative claim: lower reconstruction MSE than a uniform 16-level grid."""
    rng = np.random.default_rng(3)
    w = rng.standard_normal(64 * 4096).astype(np.float32)
    packed, absmax = oracle_mod.quantize(w)
    wn = oracle_mod.dequantize(packed, None, absmax, None, w.size)
    c1 = np.repeat(absmax, 64)
    levels = np.arange(16) / 7.5 - 1.0  # 16 uniform levels on [-1, 1]
    idx = np.clip(np.round((w / c1 + 1.0) * 7.5), 0, 15).astype(int)
    wu = levels[idx] * c1
    assert np.mean((w - wn) ** 2) < np.mean((w - wu) ** 2)
