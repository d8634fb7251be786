"""Pins of the oracle's backward pass through the frozen base.

"QLoRA: Mathematical Foundations ...", section "Gradient Computation": the
gradients of the adapter and of the input, dx = g dequant(W) + s (g B) A,
dA = s (g B)^T x, dB = s g^T (x A^T) in the weight layout W[N, K], A[r, K],
B[N, r] (the pages write L1 = A^T, L2 = B^T, W as d_in x d_out).

The pins do not retype those formulas: the forward y(x, A, B) of the oracle
(pinned on its own against numpy products) is linear in x and bilinear in
(A, B), so for any direction E the backward must satisfy the adjoint
identities
    <g, y(x)>            = <dx, x>      (y with the weight and adapter terms)
    <g, s (x E^T) B^T>   = <dA, E>
    <g, s (x A^T) F^T>   = <dB, F>
in exact arithmetic; both sides are formed in binary64 here.  Non-square
shapes (M != N != K != r) catch transposed operands; s = 0 and the zero
adapter reduce dx to a numpy product with the dequantized bf16 weight.
"""
import numpy as np
import torch

import nf4_workloads as wl

M, K, N, R, S = 12, 192, 40, 16, 1.5


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def setup(seed=21):
    c = wl.LinearCase("bwd", M, K, N, R, S, seed)
    W, x, A, B = wl.linear_inputs(c)
    g = torch.Generator().manual_seed(seed + 1)
    dy = torch.randn(M, N, generator=g).to(torch.bfloat16)
    return W, x, A, B, dy


def quantized(oracle_mod, W):
    packed, c1 = oracle_mod.quantize(bits(W).ravel())
    codes, c2, mu = oracle_mod.double_quantize(c1)
    return packed, codes, c2, mu


def test_dx_is_the_adjoint_of_the_forward(oracle_mod):
    W, x, A, B, dy = setup()
    q = quantized(oracle_mod, W)
    y = oracle_mod.lora_linear(bits(x), K, N, *q, bits(A), bits(B), R, S)          # [M, N] fp64
    dx = oracle_mod.lora_linear_bwd(bits(dy), None, K, N, *q, bits(A), bits(B), R, S, want=("dx",))["dx"]
    lhs = float(np.sum(f64(bits(dy)) * y))
    rhs = float(np.sum(dx * f64(bits(x))))
    assert abs(lhs - rhs) <= 1e-9 * (abs(lhs) + np.sum(np.abs(f64(bits(dy)) * y)))


def test_dA_and_dB_are_adjoint_to_the_adapter_terms(oracle_mod):
    W, x, A, B, dy = setup(31)
    q = quantized(oracle_mod, W)
    out = oracle_mod.lora_linear_bwd(bits(dy), bits(x), K, N, *q, bits(A), bits(B), R, S)
    assert out["dA"].shape == (R, K) and out["dB"].shape == (N, R)
    zero = (np.full(N * K // 2, 0x77, np.uint8), None, np.zeros(N * K // 64, np.float32), None)  # W = 0
    g = torch.Generator().manual_seed(99)
    E = (torch.randn(R, K, generator=g) * 0.01).to(torch.bfloat16)
    F = (torch.randn(N, R, generator=g) * 0.01).to(torch.bfloat16)
    gy = f64(bits(dy))
    yE = oracle_mod.lora_linear(bits(x), K, N, *zero, bits(E), bits(B), R, S)   # s (x E^T) B^T
    yF = oracle_mod.lora_linear(bits(x), K, N, *zero, bits(A), bits(F), R, S)   # s (x A^T) F^T
    for y, grad, direction in ((yE, out["dA"], E), (yF, out["dB"], F)):
        lhs = float(np.sum(gy * y))
        rhs = float(np.sum(grad * f64(bits(direction))))
        assert abs(lhs - rhs) <= 1e-9 * np.sum(np.abs(gy * y))


def test_zero_scaling_dx_is_a_plain_product(oracle_mod):
    W, x, A, B, dy = setup(41)
    q = quantized(oracle_mod, W)
    dx = oracle_mod.lora_linear_bwd(bits(dy), None, K, N, *q, bits(A), bits(B), R, 0.0, want=("dx",))["dx"]
    wb = oracle_mod.dequantize(*q, N * K, "bf16").reshape(N, K)
    assert np.allclose(dx, f64(bits(dy)) @ f64(wb), rtol=1e-12, atol=1e-12)


def test_rows_subset(oracle_mod):
    W, x, A, B, dy = setup(51)
    q = quantized(oracle_mod, W)
    full = oracle_mod.lora_linear_bwd(bits(dy), None, K, N, *q, bits(A), bits(B), R, S, want=("dx",))["dx"]
    rows = np.array([11, 0, 5])
    sub = oracle_mod.lora_linear_bwd(bits(dy), None, K, N, *q, bits(A), bits(B), R, S, rows=rows,
                                     want=("dx",))["dx"]
    assert np.array_equal(sub, full[rows])
