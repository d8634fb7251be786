"""Pins of the oracle's frozen-base LoRA linear.

"QLoRA: Mathematical Foundations ...", section "Forward Pass Computation":
Y = X dequant(W) + (alpha/r)(X L1) L2 with bf16 compute.  In weight layout
(W[N, K], A[r, K], B[N, r]): y = x W~^T + s (x A^T) B^T.  Special cases that
reduce to library routines pin the indexing: s = 0 is a plain matrix product
with the dequantized bf16 weight (numpy matmul), an all-zero weight leaves
only the low-rank term (two numpy matmuls), and a single row equals the
matching row of a larger batch.  Non-square shapes catch transposed operands.
"""
import numpy as np
import torch

import nf4_workloads as wl


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(bf16_bits: np.ndarray) -> np.ndarray:
    return (bf16_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def quantized(oracle_mod, W):
    packed, c1 = oracle_mod.quantize(bits(W).ravel())
    codes, c2, mu = oracle_mod.double_quantize(c1)
    return packed, codes, c2, mu


CASE = wl.LinearCase("small linear", 24, 192, 80, 16, 2.0, 11)


def test_zero_scaling_is_plain_matmul(oracle_mod):
    W, x, A, B = wl.linear_inputs(CASE)
    packed, codes, c2, mu = quantized(oracle_mod, W)
    y = oracle_mod.lora_linear(bits(x), CASE.K, CASE.N, packed, codes, c2, mu, bits(A), bits(B), CASE.r, 0.0)
    wb = oracle_mod.dequantize(packed, codes, c2, mu, CASE.N * CASE.K, "bf16").reshape(CASE.N, CASE.K)
    ref = f64(bits(x)) @ f64(wb).T
    assert y.shape == (CASE.M, CASE.N)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    y0 = oracle_mod.lora_linear(bits(x), CASE.K, CASE.N, packed, codes, c2, mu, None, None, 0, 2.0)
    assert np.allclose(y0, ref, rtol=1e-12, atol=1e-12)


def test_zero_weight_leaves_low_rank_term(oracle_mod):
    W, x, A, B = wl.linear_inputs(CASE)
    Wz = torch.zeros_like(W)
    packed, codes, c2, mu = quantized(oracle_mod, Wz)
    assert np.all(packed == 0x77)
    y = oracle_mod.lora_linear(bits(x), CASE.K, CASE.N, packed, codes, c2, mu, bits(A), bits(B), CASE.r, CASE.scaling)
    ref = CASE.scaling * ((f64(bits(x)) @ f64(bits(A)).T) @ f64(bits(B)).T)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-14)


def test_full_formula_and_row_selection(oracle_mod):
    W, x, A, B = wl.linear_inputs(CASE)
    packed, codes, c2, mu = quantized(oracle_mod, W)
    y = oracle_mod.lora_linear(bits(x), CASE.K, CASE.N, packed, codes, c2, mu, bits(A), bits(B), CASE.r, CASE.scaling)
    wb = oracle_mod.dequantize(packed, codes, c2, mu, CASE.N * CASE.K, "bf16").reshape(CASE.N, CASE.K)
    xf = f64(bits(x))
    ref = xf @ f64(wb).T + CASE.scaling * ((xf @ f64(bits(A)).T) @ f64(bits(B)).T)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    rows = np.array([5, 0, 23], np.int64)
    ys = oracle_mod.lora_linear(bits(x), CASE.K, CASE.N, packed, codes, c2, mu, bits(A), bits(B), CASE.r,
                                CASE.scaling, rows=rows)
    assert np.array_equal(ys, y[rows])
