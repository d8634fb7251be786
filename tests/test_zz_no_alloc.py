"""GPU test of nf4_lora_linear_fwd_noalloc, the fused linear for callers that
cannot allocate device memory (plugins handed only their buffers, serving
loops that must not call cudaMalloc mid-step, frameworks whose memory is
reserved by their own pool).  Its output must match nf4_lora_linear_fwd (the
entry point with a caller workspace) and the CPU oracle within the matmul
tolerance, on two calls in a row (the shared scratch keeps the previous
call's contents), and write nothing outside its output.

Collected last on purpose, so a run that stops at the first failure has
already run every other test; it also passes alone in a fresh process."""
import numpy as np
import pytest
import torch

import nf4_workloads as wl
from conftest import MATMUL_MAX_REL, MATMUL_MEAN_REL, check_guards, guarded, rel_error_stats

pytestmark = pytest.mark.gpu


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("M,K,N,r", [(16, 4096, 1024, 16), (12, 2048, 4096, 0), (300, 1024, 512, 64),
                                     (64, 512, 256, 0), (5, 1024, 640, 32)])
def test_noalloc_matches_workspace_entry_point(nf4lib, oracle_mod, cuda_device, M, K, N, r):
    c = wl.LinearCase("noalloc", M, K, N, r, 1.25, 200 + M)
    W, x, A, B = wl.linear_inputs(c, with_lora=r > 0)
    st = nf4lib.quantize_weight(W.to(cuda_device))
    xd = x.to(cuda_device)
    Ad = None if A is None else A.to(cuda_device)
    Bd = None if B is None else B.to(cuda_device)
    ref = nf4lib.nf4_lora_linear_fwd(xd, st.packed, st.absmax_q, st.absmax2, st.offset, N, Ad, Bd, c.scaling)
    # the oracle (fp64) on the same quantized weight and inputs
    exact = oracle_mod.lora_linear(u16(x), K, N, st.packed.cpu().numpy(), st.absmax_q.cpu().numpy(),
                                   st.absmax2.cpu().numpy(), np.float32(st.offset.cpu().numpy()[0]),
                                   None if A is None else u16(A), None if B is None else u16(B), r, c.scaling)
    for _ in range(2):
        y = guarded((M, N), torch.bfloat16, cuda_device, fill=float("nan"))
        nf4lib.nf4_lora_linear_fwd_noalloc(xd, st.packed, st.absmax_q, st.absmax2, st.offset, N, Ad, Bd,
                                          c.scaling, y=y)
        nf4lib.nf4_device_status()
        check_guards(y)
        got = y.float().cpu().numpy()
        mx, mean, _ = rel_error_stats(got, ref.float().cpu().numpy())
        assert mx <= MATMUL_MAX_REL and mean < MATMUL_MEAN_REL, (mx, mean)
        mx, mean, _ = rel_error_stats(got, exact)
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
