"""Pins of the oracle's merge of the adapter into the quantized base and the
requantization that follows.

"QLoRA in Production ...", section "Step 4: Merging and Inference" (merge the
adapter into the quantized base), and "QLoRA: quantising the part you are not
training", section "What it costs" ("Merging is awkward": a merge into the
quantized base has to be requantized).  Reading (the pages give no
arithmetic): W' = fma(s, d, w~) in binary32, d the fused chain
d <- fma(B[n, j], A[j, k], d) over j in order.  Pins: the delta against an
fp64 matrix product (non-square shapes catch a transposed operand), s = 0
giving back the dequantized weight, requantizing an unmerged weight giving
back its codes and its reconstructed constants (a property of the format),
and an exact-rational re-evaluation of a tiny case with a brute-force
nearest-level search.
"""
from fractions import Fraction

import numpy as np
import torch

import nf4_workloads as wl
from numerics import fma_f32

N, K, R = 48, 320, 24


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def adapter(seed, n=N, k=K, r=R, sigma=0.05):
    g = torch.Generator().manual_seed(seed)
    A = (torch.randn(r, k, generator=g) * sigma).to(torch.bfloat16)
    B = (torch.randn(n, r, generator=g) * sigma).to(torch.bfloat16)
    return bits(A), bits(B)


def quantized(oracle_mod, W, dq=True):
    packed, c1 = oracle_mod.quantize(bits(W).ravel())
    if not dq:
        return packed, None, c1, None
    codes, c2, mu = oracle_mod.double_quantize(c1)
    return packed, codes, c2, mu


def test_delta_on_a_zero_weight_is_the_scaled_product(oracle_mod):
    A, B = adapter(1)
    packed = np.full(N * K // 2, 0x77, np.uint8)  # every code 7 (level 0)
    c1 = np.zeros(N * K // 64, np.float32)
    s = 0.75
    got = oracle_mod.merge_weight(packed, None, c1, None, K, A, B, R, s).astype(np.float64)
    prod = f64(B) @ f64(A)                      # [N, K] = B A
    ref = s * prod
    bound = (R + 2) * 2.0 ** -24 * s * (np.abs(f64(B)) @ np.abs(f64(A))) + 1e-30
    assert got.shape == (N, K)
    assert np.all(np.abs(got - ref) <= bound)


def test_zero_scaling_gives_back_the_dequantized_weight(oracle_mod):
    W = wl.weight((N, K), 0.02, 7, "bf16")
    packed, codes, c2, mu = quantized(oracle_mod, W)
    A, B = adapter(2)
    got = oracle_mod.merge_weight(packed, codes, c2, mu, K, A, B, R, 0.0)
    deq = oracle_mod.dequantize(packed, codes, c2, mu, N * K, "f32").reshape(N, K)
    assert np.array_equal(got, deq)


def test_requantizing_an_unmerged_weight_returns_its_codes(oracle_mod):
    W = wl.weight((N, K), 0.02, 8, "bf16", outliers=True)
    for dq in (True, False):
        packed, codes, sc, mu = quantized(oracle_mod, W, dq)
        A, B = adapter(3)
        pk, ab = oracle_mod.merge_requantize(packed, codes, sc, mu, K, A, B, R, 0.0)
        deq = oracle_mod.dequantize(packed, codes, sc, mu, N * K, "f32").reshape(-1, 64)
        c1r = np.max(np.abs(deq), axis=1)   # reconstructed constants c1'
        assert np.all(c1r > 0)
        assert np.array_equal(ab, c1r.astype(np.float32))
        assert np.array_equal(pk, packed)


def test_rows_subset_matches_full(oracle_mod):
    W = wl.weight((N, K), 0.02, 9, "bf16")
    packed, codes, c2, mu = quantized(oracle_mod, W)
    A, B = adapter(4)
    full_p, full_a = oracle_mod.merge_requantize(packed, codes, c2, mu, K, A, B, R, 1.5)
    p, a = oracle_mod.merge_requantize(packed, codes, c2, mu, K, A, B, R, 1.5, row0=17, nrows=9)
    assert np.array_equal(p, full_p[17 * K // 2:26 * K // 2])
    assert np.array_equal(a, full_a[17 * K // 64:26 * K // 64])


def nearest_code(x: np.float32, levels) -> int:
    """Brute-force arg-min of |x - q_i| with exact rational distances, lower
    index on ties."""
    fx = Fraction(float(x))
    best = None
    for i, q in enumerate(levels):
        d = abs(fx - Fraction(float(q)))
        if best is None or d < best[0]:
            best = (d, i)
    return best[1]


def test_tiny_case_exactly(oracle_mod):
    n, k, r, s = 2, 64, 3, np.float32(1.25)
    W = wl.weight((n, k), 0.02, 10, "bf16")
    packed, c1 = oracle_mod.quantize(bits(W).ravel())  # no double quantization
    A, B = adapter(5, n, k, r, sigma=0.02)
    levels = oracle_mod.codebook()
    deq = oracle_mod.dequantize(packed, None, c1, None, n * k, "f32").reshape(n, k)
    Af, Bf = f64(A).astype(np.float32), f64(B).astype(np.float32)
    ref = np.empty((n, k), np.float32)
    for i in range(n):
        for j in range(k):
            d = np.float32(0.0)
            for q in range(r):
                d = fma_f32(Bf[i, q], Af[q, j], d)
            ref[i, j] = fma_f32(s, d, deq[i, j])
    got = oracle_mod.merge_weight(packed, None, c1, None, k, A, B, r, float(s))
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))
    pk, ab = oracle_mod.merge_requantize(packed, None, c1, None, k, A, B, r, float(s))
    for i in range(n):
        blk = ref[i]
        c = np.float32(np.max(np.abs(blk)))
        assert ab[i] == c
        for j in range(k):
            code = nearest_code(np.float32(blk[j] / c), levels)  # binary32 quotient
            nib = (pk[(i * k + j) >> 1] >> 4) if (j % 2 == 0) else (pk[(i * k + j) >> 1] & 15)
            assert nib == code
