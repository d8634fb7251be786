"""NF4 (QLoRA 4-bit NormalFloat) quantization and the fused frozen-base LoRA
linear on NVIDIA B200: a C-ABI CUDA library (libnf4.so, include/nf4.h) and a
thin ctypes binding with the same entry-point names.

Every step runs in the library's sm_100a kernels; PyTorch only provides
device memory and streams.  Importing the binding fails loudly if libnf4.so
has not been built (``python -m qlora_nf4_quantize_b200.build``).
"""
from .nf4 import (  # noqa: F401
    BLOCKSIZE, DQ_BLOCKSIZE, Nf4Error, lib, nf4_codebook, nf4_quantize, nf4_double_quantize,
    nf4_double_quantize_workspace_size, nf4_dequantize, nf4_lora_linear_fwd,
    nf4_lora_linear_workspace_size, nf4_lora_linear_fwd_noalloc, nf4_device_status, nf4_selftest_wait_timeout, nf4_merge_requantize, nf4_lora_linear_bwd,
    nf4_lora_linear_bwd_workspace_size, nf4_dq_run_sums, nf4_double_quantize_sharded, nf4_quantize_dq,
    nf4_quantize_dq_workspace_size, QuantState,
    quantize_weight, merge_and_requantize,
)
from . import sharded  # noqa: F401
