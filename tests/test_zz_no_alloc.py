"""GPU test of nf4_lora_linear_fwd_noalloc, the fused linear for callers that
cannot allocate device memory (plugins handed only their buffers, serving
loops that must not call cudaMalloc mid-step, frameworks whose memory is
reserved by their own pool).  Its output must match nf4_lora_linear_fwd (the
entry point with a caller workspace) within the matmul tolerance, on two
calls in a row (the shared scratch keeps the previous call's contents;
up to 16 tokens it also holds the split pipeline's partial tiles and
arrival counts).

Collected last on purpose, so a run that stops at the first failure has
already run every other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import nf4_workloads as wl
from conftest import MATMUL_MAX_REL, MATMUL_MEAN_REL, rel_error_stats

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K,N,r", [(16, 4096, 1024, 16), (12, 2048, 4096, 0), (300, 1024, 512, 64),
                                     (64, 512, 256, 0)])
def test_noalloc_matches_workspace_entry_point(nf4lib, cuda_device, M, K, N, r):
    c = wl.LinearCase("noalloc", M, K, N, r, 1.25, 200 + M)
    W, x, A, B = wl.linear_inputs(c, with_lora=r > 0)
    st = nf4lib.quantize_weight(W.to(cuda_device))
    xd = x.to(cuda_device)
    Ad = None if A is None else A.to(cuda_device)
    Bd = None if B is None else B.to(cuda_device)
    ref = nf4lib.nf4_lora_linear_fwd(xd, st.packed, st.absmax_q, st.absmax2, st.offset, N, Ad, Bd, c.scaling)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=cuda_device)
        nf4lib.nf4_lora_linear_fwd_noalloc(xd, st.packed, st.absmax_q, st.absmax2, st.offset, N, Ad, Bd,
                                          c.scaling, y=y)
        nf4lib.nf4_device_status()
        mx, mean, _ = rel_error_stats(y.float().cpu().numpy(), ref.float().cpu().numpy())
        assert mx <= MATMUL_MAX_REL and mean < MATMUL_MEAN_REL, (mx, mean)


def test_noalloc_rejects_sizes_beyond_the_scratch(nf4lib, cuda_device):
    x = torch.zeros(16385, 64, dtype=torch.bfloat16, device=cuda_device)
    packed = torch.zeros(64 * 64 // 2, dtype=torch.uint8, device=cuda_device)
    absmax = torch.zeros(64, dtype=torch.float32, device=cuda_device)
    A = torch.zeros(64, 64, dtype=torch.bfloat16, device=cuda_device)
    B = torch.zeros(64, 64, dtype=torch.bfloat16, device=cuda_device)
    y = torch.empty(16385, 64, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(nf4lib.Nf4Error, match="NF4_ERR_UNSUPPORTED"):
        nf4lib.nf4_lora_linear_fwd_noalloc(x, packed, None, absmax, None, 64, A, B, 1.0, y=y)
