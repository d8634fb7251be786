"""Failure detection on the GPU without a fault: a bounded wait that nothing
satisfies expires, the kernel raises the library's device error word and
returns, the host reads NF4_ERR_TIMEOUT from nf4_device_status, and the
context stays usable (a normal call afterwards is still exact)."""
import time

import pytest
import torch

import nf4_workloads as wl

pytestmark = pytest.mark.gpu

NF4_ERR_TIMEOUT = 4


def test_expired_wait_is_reported_and_cleared(nf4lib, oracle_mod, cuda_device):
    nf4lib.nf4_device_status()  # start from a clear error word
    t0 = time.perf_counter()
    nf4lib.nf4_selftest_wait_timeout(20_000_000)  # 20 ms
    with pytest.raises(nf4lib.Nf4Error) as ei:
        nf4lib.nf4_device_status()
    elapsed = time.perf_counter() - t0
    assert ei.value.status == NF4_ERR_TIMEOUT
    assert elapsed >= 0.02
    assert nf4lib.nf4_device_status() == 0  # the word was cleared

    # the context is still usable: a quantize / dequantize round trip stays exact
    w = wl.weight_case(wl.TINY).to(cuda_device).reshape(-1)
    packed, absmax = nf4lib.nf4_quantize(w)
    out = nf4lib.nf4_dequantize(packed, None, absmax, None, w.numel(), torch.float32)
    torch.cuda.synchronize()
    bits = w.cpu().numpy()
    p_ref, c_ref = oracle_mod.quantize(bits)
    assert (packed.cpu().numpy() == p_ref).all()
    assert (out.cpu().numpy() == oracle_mod.dequantize(p_ref, None, c_ref, None, w.numel(), "f32")).all()
