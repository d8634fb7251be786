"""Pins of the oracle's double quantization and storage arithmetic.

"QLoRA: Mathematical Foundations ...", section "Double Quantization (DQ)":
runs of 256 first-level constants, c2 = max |c1| per run, 8-bit float codes of
c1 / c2.  READINGS (format E4M3 round-to-nearest-even, a per-tensor mean mu
subtracted first, fixed-order fp64 sum for mu) are pinned where the
mathematics fixes them: the E4M3 encoder and decoder against torch's
float8_e4m3fn casts (library routine), c2 against the exact maximum, mu
against the exact rational mean where the fp64 sums are exact, and the
reconstruction error against the E4M3 spacing.  The summation order of mu is
a convention: parity unpinned against the pages (pinned oracle-vs-GPU only).
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import nf4_workloads as wl
from conftest import read_golden_kv
from numerics import fma_f32


def e4m3_all_finite_values():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_e4m3_decode_all_codes(oracle_mod):
    ref = e4m3_all_finite_values()
    for c in range(256):
        got = oracle_mod.e4m3_decode(c)
        if math.isnan(ref[c]):
            assert math.isnan(got)
        else:
            assert got == ref[c] and math.copysign(1, got) == math.copysign(1, ref[c])


def torch_e4m3(y: np.ndarray) -> np.ndarray:
    return torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_against_library(oracle_mod):
    vals = e4m3_all_finite_values()
    pos = np.unique(vals[(vals >= 0) & np.isfinite(vals) & (vals <= 1.0)])
    probes = [np.float32(0.0), np.float32(-0.0)]
    for a, b in zip(pos[:-1], pos[1:]):
        m = np.float32((a + b) / 2)  # midpoints are exact in binary32 here
        v = m
        for _ in range(3):
            v = np.nextafter(v, np.float32(-2))
        for _ in range(7):
            probes.append(v)
            v = np.nextafter(v, np.float32(2))
    probes += list(pos.astype(np.float32))
    rng = np.random.default_rng(5)
    probes = np.array(probes, np.float32)
    probes = np.concatenate([probes, -probes, rng.uniform(-1, 1, 200000).astype(np.float32),
                             (rng.uniform(-1, 1, 20000) * 2.0 ** -8).astype(np.float32)])
    assert np.array_equal(oracle_mod.e4m3_encode_array(probes), torch_e4m3(probes))


def test_e4m3_encode_saturates(oracle_mod):
    assert oracle_mod.e4m3_encode(1000.0) == 0x7E
    assert oracle_mod.e4m3_encode(-1000.0) == 0xFE
    assert oracle_mod.e4m3_encode(448.0) == 0x7E


def exact_mean_f32(vals):
    s = sum(Fraction(float(v)) for v in vals)
    return np.float32(float(s / len(vals)))  # float() rounds the rational to nearest binary64


def test_dq_mean_equals_exact_mean_when_sums_are_exact(oracle_mod):
    # constants of one magnitude range: every fp64 partial sum is exact, so mu is
    # RN_f32(RN_f64(exact mean)) regardless of order
    rng = np.random.default_rng(7)
    for nb in (1, 2, 255, 256, 257, 2048, 5000):
        c1 = (rng.uniform(0.01, 0.1, nb)).astype(np.float32)
        assert oracle_mod.dq_mean(c1) == exact_mean_f32(c1)


def test_double_quantize_scales_and_codes(oracle_mod):
    w = wl.weight_case(wl.TINY).numpy().ravel()
    _, c1 = oracle_mod.quantize(w)
    codes, c2, mu = oracle_mod.double_quantize(c1)
    assert c1.size == 2048 and c2.size == 8 and codes.size == 2048
    d = (c1 - mu).astype(np.float32)
    for k in range(8):
        assert c2[k] == np.max(np.abs(d[k * 256:(k + 1) * 256]))
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    rec = dec.astype(np.float64) * np.repeat(c2, 256).astype(np.float64) + float(mu)
    # E4M3 in [-1, 1]: relative step 2^-3 for normals, absolute 2^-9 subnormal
    y = d.astype(np.float64) / np.repeat(c2, 256)
    tol = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * np.repeat(c2, 256) + np.abs(rec) * 2.0 ** -23
    assert np.all(np.abs(rec - c1) <= tol)


def test_double_quantize_without_centring_is_literal_formula(oracle_mod):
    rng = np.random.default_rng(8)
    c1 = rng.uniform(0.0, 0.2, 700).astype(np.float32)
    codes, c2, mu = oracle_mod.double_quantize(c1, centre=False)
    assert mu == 0.0
    for k in range(c2.size):
        blk = c1[k * 256:(k + 1) * 256]
        assert c2[k] == np.max(blk)
        want = torch_e4m3((blk / c2[k]).astype(np.float32))
        assert np.array_equal(codes[k * 256:(k + 1) * 256], want)


def test_centred_codes_bit_for_bit(oracle_mod):
    """Centred codes are E4M3 (torch.float8_e4m3fn, a library routine) of
    RN(RN(c1 - mu) / c2), each step one binary32 rounding (numpy float32
    arithmetic), with c2 the run's max |RN(c1 - mu)|; a run with c2 = 0 stores
    0.  Constants from the projection weight (outliers included) and a mix of
    magnitudes on both sides of the mean."""
    _, proj = oracle_mod.quantize(wl.weight_case(wl.PROJECTION).float().numpy().ravel())
    rng = np.random.default_rng(17)
    mixed = (rng.uniform(0.0, 1.0, 256 * 9 + 77) * 2.0 ** rng.integers(-12, 3, 256 * 9 + 77)).astype(np.float32)
    mixed[256 * 2:256 * 3] = np.float32(0.25)  # a run near the mean of its neighbours
    for c1 in (proj, mixed):
        codes, c2, mu = oracle_mod.double_quantize(c1)
        d = c1 - np.float32(mu)
        assert d.dtype == np.float32
        for k in range(c2.size):
            dk = d[k * 256:(k + 1) * 256]
            assert c2[k] == np.max(np.abs(dk))
            if c2[k] == 0:
                want = np.zeros(dk.size, np.uint8)
            else:
                y = dk / np.float32(c2[k])
                assert y.dtype == np.float32
                want = torch_e4m3(y)
            assert np.array_equal(codes[k * 256:(k + 1) * 256], want), k

def test_double_quantize_zero_run(oracle_mod):
    c1 = np.full(300, 0.05, np.float32)  # every constant equal to the mean
    codes, c2, mu = oracle_mod.double_quantize(c1)
    assert mu == np.float32(0.05)
    assert np.all(c2 == 0) and np.all(codes == 0)


def test_dq_dequantize_round_trip_bound(oracle_mod):
    """|w - w~| <= |q| |c1 - c1'| + c1 (g/2 + 2^-22) with DQ."""
    w = wl.weight_case(wl.TINY).numpy().ravel()
    packed, c1 = oracle_mod.quantize(w)
    codes, c2, mu = oracle_mod.double_quantize(c1)
    wt = oracle_mod.dequantize(packed, codes, c2, mu, w.size)
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    c1p = np.array([fma_f32(a, b, mu) for a, b in zip(dec, np.repeat(c2, 256))], np.float32)
    q = oracle_mod.codebook()
    cd = np.empty(w.size, np.int64)
    cd[0::2] = packed >> 4
    cd[1::2] = packed & 15
    # exact: w~ = RN(q * c1')
    assert np.array_equal(wt, q[cd] * np.repeat(c1p, 64))
    gaps = np.maximum(np.diff(q, prepend=q[0]), np.diff(q, append=q[-1])).astype(np.float64)
    c1r = np.repeat(c1.astype(np.float64), 64)
    bound = np.abs(q[cd]) * np.abs(c1r - np.repeat(c1p.astype(np.float64), 64)) + c1r * (gaps[cd] / 2 + 2.0 ** -22)
    assert np.all(np.abs(w - wt.astype(np.float64)) <= bound + 1e-12)


def storage_bytes(n, bs=64, dqbs=256, dq=True):
    nb = -(-n // bs)
    nd = -(-nb // dqbs)
    return n // 2 + (nb + 4 * nd + 4 if dq else 4 * nb)


def test_output_sizes_match_closed_forms(oracle_mod):
    g = read_golden_kv("storage_arithmetic.txt")
    w = wl.weight_case(wl.TINY).numpy().ravel()
    packed, c1 = oracle_mod.quantize(w)
    codes, c2, _ = oracle_mod.double_quantize(c1)
    n = w.size
    assert packed.nbytes + codes.nbytes + c2.nbytes + 4 == storage_bytes(n)
    assert packed.nbytes + c1.nbytes == storage_bytes(n, dq=False)
    # per-parameter figures (one DQ run = 64 * 256 = 16384 parameters)
    assert 64 * 256 == g["params_per_dq_block"]
    per_param_dq = (packed.nbytes + codes.nbytes + c2.nbytes) / n
    per_param_nodq = (packed.nbytes + c1.nbytes) / n
    assert per_param_nodq == g["bytes_per_param_no_dq"]
    assert per_param_dq == 0.5 + 1 / 64 + 4 / 16384
    assert round(per_param_dq, 4) == g["bytes_per_param_dq"]
    assert round(per_param_dq * 8, 2) == g["bits_per_param_dq"]
    scale_bits = (codes.nbytes + c2.nbytes) * 8 / n
    assert c1.nbytes * 8 / n == g["scale_bits_per_param_no_dq"]
    assert round(scale_bits, 3) == g["scale_bits_per_param_dq"]
    assert round(scale_bits * 64, 3) == g["scale_bits_per_block_dq"]
    assert round(0.5 - round(scale_bits, 3), 3) == g["dq_saving_bits_per_param"]
    assert round(100 * (0.5 - 0.127) / 0.5, 1) == g["dq_saving_percent"]


def test_page_model_scale_figures():
    g = read_golden_kv("storage_arithmetic.txt")
    assert round(7e9 / 64 / 1e6, 1) == g["blocks_7b_millions"]
    assert round(7e9 / 64 * 4 / 1e6, 1) == g["scale_bytes_7b_mb"]
    # 65B: saving of (0.5 - 0.127) bits per parameter, in GB (1e9 bytes)
    assert round(65e9 * (0.5 - 0.127) / 8 / 1e9, 2) == g["dq_saving_65b_gb"]
    per_param = 0.5 + 1 / 64 + 4 / 16384
    assert round(8e9 * 2 / 1e9) == g["footprint_8b_bf16_gb"]
    assert round(8e9 * per_param / 1e9, 1) == g["footprint_8b_nf4_gb"]
    assert round(70e9 * 2 / 1e9) == g["footprint_70b_bf16_gb"]
    assert round(70e9 * per_param / 1e9) == g["footprint_70b_nf4_gb"]


def test_8b_shaped_sweep_storage():
    n_linear = sum(N * K for _, N, K in wl.LAYER_8B) * wl.N_LAYERS_8B
    assert n_linear == 6_979_321_856
    total = sum(storage_bytes(N * K) for _, N, K in wl.LAYER_8B) * wl.N_LAYERS_8B
    assert total == 3_600_416_768 + 4 * 7 * 32
