"""GPU parity of nf4_merge_requantize (merge the adapter into the quantized
base and requantize) against the oracle: packed codes and fp32 block
constants bit-exact, and the double quantization of the result bit-exact too.

"QLoRA in Production ...", section "Step 4: Merging and Inference";
"QLoRA: quantising the part you are not training", section "What it costs"
(item 3).  The merge arithmetic is the reading stated in include/nf4.h."""
import numpy as np
import pytest
import torch

import nf4_workloads as wl
from conftest import check_guards, guarded

pytestmark = pytest.mark.gpu


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def case(N, K, r, seed):
    g = torch.Generator().manual_seed(seed)
    W = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16)
    A = (torch.randn(max(r, 1), K, generator=g) * 0.02).to(torch.bfloat16)[:r]
    B = (torch.randn(N, max(r, 1), generator=g) * 0.02).to(torch.bfloat16)[:, :r].contiguous()
    return W, A, B


def state_np(st):
    return (st.packed.cpu().numpy(), None if st.absmax_q is None else st.absmax_q.cpu().numpy(),
            st.absmax2.cpu().numpy(), None if st.offset is None else float(st.offset.cpu().numpy()[0]))


@pytest.mark.parametrize("N,K,r,mode", [(200, 320, 16, "dq"), (64, 256, 64, "nodq"), (130, 192, 32, "uncentred"),
                                        (48, 4096, 7, "dq"), (33, 64, 0, "dq"), (70, 640, 64, "dq"),
                                        (96, 128, 8, "dq"), (80, 512, 24, "nodq")])
def test_merge_requantize_bit_exact(nf4lib, oracle_mod, cuda_device, N, K, r, mode):
    W, A, B = case(N, K, r, 1000 + N + K + r)
    st = nf4lib.quantize_weight(W.to(cuda_device), double_quant=(mode != "nodq"), centre=(mode == "dq"))
    s = 1.75
    Ad = A.to(cuda_device) if r else None
    Bd = B.to(cuda_device) if r else None
    pk, ab = guarded(N * K // 2, torch.uint8, cuda_device), guarded(N * K // 64, torch.float32, cuda_device)
    nf4lib.nf4_merge_requantize(st.packed, st.absmax_q, st.absmax2, st.offset, N, K, Ad, Bd, s, packed_out=pk,
                                absmax_out=ab)
    torch.cuda.synchronize()
    check_guards(pk, ab)
    packed, codes, sc, mu = state_np(st)
    ref_p, ref_a = oracle_mod.merge_requantize(packed, codes, sc, mu, K, bits(A) if r else None,
                                               bits(B) if r else None, r, s)
    assert np.array_equal(pk.cpu().numpy(), ref_p)
    assert np.array_equal(ab.cpu().numpy().view(np.uint32), ref_a.view(np.uint32))
    # back to the stored format: double quantization of the new constants
    q8, c2, off = nf4lib.nf4_double_quantize(ab)
    r8, rc2, rmu = oracle_mod.double_quantize(ref_a)
    assert np.array_equal(q8.cpu().numpy(), r8)
    assert np.array_equal(c2.cpu().numpy().view(np.uint32), rc2.view(np.uint32))
    assert np.float32(off.cpu().numpy()[0]).view(np.uint32) == np.float32(rmu).view(np.uint32)


def test_merge_in_place(nf4lib, oracle_mod, cuda_device):
    N, K, r = 96, 512, 16
    W, A, B = case(N, K, r, 77)
    pk, ab = guarded(N * K // 2, torch.uint8, cuda_device), guarded(N * K // 64, torch.float32, cuda_device)
    nf4lib.nf4_quantize(W.to(cuda_device).reshape(-1), packed=pk, absmax=ab)
    st = nf4lib.QuantState(pk, None, ab, None, (N, K))
    packed, codes, sc, mu = state_np(st)
    nf4lib.nf4_merge_requantize(st.packed, None, st.absmax2, None, N, K, A.to(cuda_device), B.to(cuda_device), 0.5,
                                packed_out=st.packed, absmax_out=st.absmax2)
    torch.cuda.synchronize()
    check_guards(pk, ab)
    ref_p, ref_a = oracle_mod.merge_requantize(packed, codes, sc, mu, K, bits(A), bits(B), r, 0.5)
    assert np.array_equal(st.packed.cpu().numpy(), ref_p)
    assert np.array_equal(st.absmax2.cpu().numpy().view(np.uint32), ref_a.view(np.uint32))


def test_merge_training_weight_sampled_rows(nf4lib, oracle_mod, cuda_device):
    c = wl.GEMM_TRAIN
    W, _, A, B = wl.linear_inputs(c)
    st = nf4lib.quantize_weight(W.to(cuda_device))
    pk, ab = guarded(c.N * c.K // 2, torch.uint8, cuda_device), guarded(c.N * c.K // 64, torch.float32, cuda_device)
    nf4lib.nf4_merge_requantize(st.packed, st.absmax_q, st.absmax2, st.offset, c.N, c.K, A.to(cuda_device),
                                B.to(cuda_device), c.scaling, packed_out=pk, absmax_out=ab)
    torch.cuda.synchronize()
    check_guards(pk, ab)
    packed, codes, sc, mu = state_np(st)
    pk, ab = pk.cpu().numpy(), ab.cpu().numpy()
    K = c.K
    for row0 in (0, 7001, c.N - 16):
        rp, ra = oracle_mod.merge_requantize(packed, codes, sc, mu, K, bits(A), bits(B), c.r, c.scaling,
                                             row0=row0, nrows=16)
        assert np.array_equal(pk[row0 * K // 2:(row0 + 16) * K // 2], rp)
        assert np.array_equal(ab[row0 * K // 64:(row0 + 16) * K // 64].view(np.uint32), ra.view(np.uint32))
