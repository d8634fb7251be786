"""Seeded synthetic inputs for the NF4 workloads.

This module only draws random numbers and names shapes; it holds none of the
method's arithmetic.  Both the CUDA path (tests, benchmark) and the CPU oracle
consume what it returns, so they always see identical inputs.

Distributions follow the pages: weights ~ N(0, sigma^2) (pretrained weight
matrices are modelled as zero-mean Gaussians on the Mathematical Foundations
page, section "4-Bit NormalFloat (NF4)"), activations ~ N(0, 1), LoRA factors
~ N(0, 0.01^2).  All draws come from a CPU ``torch.Generator`` in the fixed
order W, outlier mask, x, A, B; bf16 tensors are the fp32 draws rounded to
nearest-even by ``Tensor.to(torch.bfloat16)``.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class LinearCase:
    name: str
    M: int
    K: int
    N: int
    r: int
    scaling: float
    seed: int
    w_sigma: float = 0.02
    lora_sigma: float = 0.01


# Workload shapes (sizes from the Llama-style layers the pages discuss).
TINY = dict(name="tiny round trip fp32 256x512", shape=(256, 512), dtype="f32", seed=0, outliers=False)
PROJECTION = dict(name="projection bf16 4096x4096 with 0.1% x10 outliers", shape=(4096, 4096),
                  dtype="bf16", seed=1, outliers=True)
GEMV_CASES = [LinearCase(f"decode GEMV T={T} W 11008x4096 r=16", T, 4096, 11008, 16, 2.0, 3)
              for T in (1, 4, 16)]
GEMM_TRAIN = LinearCase("training GEMM x 4096x4096, W 14336x4096, r=64", 4096, 4096, 14336, 64, 0.25, 4)
GEMM_70B_MLP = LinearCase("70B MLP GEMM x 2048x8192, W 28672x8192, r=16", 2048, 8192, 28672, 16, 2.0, 5)
# Two more linears of the 8B-shaped decoder layer at the training token count
# (the layer's longest contraction and its narrowest output)
GEMM_DOWN_PROJ = LinearCase("down_proj GEMM x 4096x14336, W 4096x14336, r=64", 4096, 14336, 4096, 64, 0.25, 6)
GEMM_K_PROJ = LinearCase("k_proj GEMM x 4096x4096, W 1024x4096, r=64", 4096, 4096, 1024, 64, 0.25, 7)

# One decoder layer of the 8B-shaped model: (name, out_features N, in_features K)
LAYER_8B = [("q_proj", 4096, 4096), ("k_proj", 1024, 4096), ("v_proj", 1024, 4096),
            ("o_proj", 4096, 4096), ("gate_proj", 14336, 4096), ("up_proj", 14336, 4096),
            ("down_proj", 4096, 14336)]
N_LAYERS_8B = 32


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def weight(shape, sigma: float, seed: int, dtype: str = "bf16", outliers: bool = False,
           outlier_rate: float = 1e-3, outlier_scale: float = 10.0) -> torch.Tensor:
    """W ~ N(0, sigma^2) of ``shape``; with ``outliers`` a fraction
    ``outlier_rate`` of entries (uniform mask drawn after W) is multiplied by
    ``outlier_scale``.  Returns a CPU tensor of dtype float32 or bfloat16."""
    g = _gen(seed)
    w = torch.randn(*shape, generator=g, dtype=torch.float32) * sigma
    if outliers:
        mask = torch.rand(*shape, generator=g, dtype=torch.float32) < outlier_rate
        w = torch.where(mask, w * outlier_scale, w)
    return w if dtype == "f32" else w.to(torch.bfloat16)


def weight_case(case: dict) -> torch.Tensor:
    return weight(case["shape"], 0.02, case["seed"], case["dtype"], case["outliers"])


def linear_inputs(c: LinearCase, with_lora: bool = True):
    """(W bf16 [N,K], x bf16 [M,K], A bf16 [r,K], B bf16 [N,r]) drawn in the
    order W, x, A, B from one generator seeded with ``c.seed``."""
    g = _gen(c.seed)
    W = (torch.randn(c.N, c.K, generator=g) * c.w_sigma).to(torch.bfloat16)
    x = torch.randn(c.M, c.K, generator=g).to(torch.bfloat16)
    if not with_lora or c.r == 0:
        return W, x, None, None
    A = (torch.randn(c.r, c.K, generator=g) * c.lora_sigma).to(torch.bfloat16)
    B = (torch.randn(c.N, c.r, generator=g) * c.lora_sigma).to(torch.bfloat16)
    return W, x, A, B


def sweep_seed(layer: int, idx: int) -> int:
    return 5 * 1000 + 7 * layer + idx


def sweep_weight(layer: int, idx: int) -> torch.Tensor:
    """Linear ``idx`` of decoder layer ``layer`` of the 8B-shaped sweep, bf16."""
    _, N, K = LAYER_8B[idx]
    return weight((N, K), 0.02, sweep_seed(layer, idx), "bf16")


def random_bits_f32(n: int, seed: int) -> torch.Tensor:
    """n arbitrary finite float32 values of mixed magnitudes (edge-case
    generator): N(0,1) scaled by 2^U with U uniform in [-40, 40]."""
    g = _gen(seed)
    base = torch.randn(n, generator=g)
    expo = torch.randint(-40, 41, (n,), generator=g).to(torch.float32)
    return base * torch.pow(2.0, expo)
