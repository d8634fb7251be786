"""GPU parity of the sharded quantization path (nf4_dq_run_sums and
nf4_double_quantize_sharded through qlora_nf4_quantize_b200.sharded): a
tensor cut into 2, 3 or 5 shards on run boundaries, each shard quantized on
its own as a rank would, the run sums concatenated in rank order (what the
all-gather delivers), and every shard double-quantized with the tensor-wide
mean.  Packed codes, constants, mu, c2 and 8-bit codes are bit-identical to
the one-shot quantization of the whole tensor and to the CPU oracle.  The
ranks run one after another on one GPU: no kernel waits on another."""
import numpy as np
import pytest
import torch

import nf4_workloads as wl
from conftest import check_guards, guarded

pytestmark = pytest.mark.gpu

RUN = 64 * 256


def u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("shape,world", [((4096, 4096), 2), ((4096, 4096), 3), ((1000, 1000), 5),
                                         ((14336, 4096), 3)])
def test_sharded_equals_one_shot_and_oracle(nf4lib, oracle_mod, cuda_device, shape, world):
    from qlora_nf4_quantize_b200 import sharded
    w = wl.weight(shape, 0.02, 900 + world, "bf16", outliers=True)
    n = w.numel()
    wd = w.to(cuda_device).reshape(-1)
    # phase 1 on every "rank": codes, constants, run sums (guarded outputs)
    local = []
    for r in range(world):
        e0, e1 = sharded.shard_range(n, world, r)
        m = e1 - e0
        pk, ab = guarded(m // 2, torch.uint8, cuda_device), guarded(-(-m // 64), torch.float32, cuda_device)
        nf4lib.nf4_quantize(wd[e0:e1], packed=pk, absmax=ab)
        sums = guarded(-(-ab.numel() // 256), torch.float64, cuda_device)
        nf4lib.nf4_dq_run_sums(ab, out=sums)
        local.append((pk, ab, sums))
    all_sums = torch.cat([s for _, _, s in local])
    # phase 2 on every "rank"
    parts = []
    for pk, ab, sums in local:
        nb = ab.numel()
        q8, c2 = guarded(nb, torch.uint8, cuda_device), guarded(-(-nb // 256), torch.float32, cuda_device)
        off = guarded(1, torch.float32, cuda_device)
        nf4lib.nf4_double_quantize_sharded(ab, all_sums, -(-n // 64), absmax_q=q8, absmax2=c2, offset=off)
        parts.append((pk, ab, q8, c2, off))
    torch.cuda.synchronize()
    for pk, ab, sums in local:
        check_guards(pk, ab, sums)
    for p in parts:
        check_guards(*p[2:])
    whole = nf4lib.quantize_weight(wd)
    packed = torch.cat([p[0] for p in parts])
    q8 = torch.cat([p[2] for p in parts])
    c2 = torch.cat([p[3] for p in parts])
    assert torch.equal(packed, whole.packed)
    assert torch.equal(q8, whole.absmax_q)
    assert torch.equal(c2.view(torch.int32), whole.absmax2.view(torch.int32))
    for p in parts:
        assert torch.equal(p[4].view(torch.int32), whole.offset.view(torch.int32))
    # and the oracle
    op, oa = oracle_mod.quantize(u16(w).ravel())
    oq8, oc2, omu = oracle_mod.double_quantize(oa)
    assert np.array_equal(packed.cpu().numpy(), op)
    assert np.array_equal(q8.cpu().numpy(), oq8)
    assert np.array_equal(c2.cpu().numpy().view(np.uint32), oc2.view(np.uint32))
    assert np.float32(parts[0][4].item()).view(np.uint32) == np.float32(omu).view(np.uint32)
    assert np.array_equal(all_sums.cpu().numpy(), oracle_mod.dq_run_sums(oa))


def test_quantize_sharded_with_a_given_gather(nf4lib, cuda_device):
    """quantize_sharded with the gather supplied by the caller (world size
    1: the rank's own sums are the whole array) equals quantize_weight."""
    from qlora_nf4_quantize_b200 import sharded
    w = wl.weight((512, 768), 0.02, 77, "bf16").to(cuda_device)
    st = sharded.quantize_sharded(w, w.numel(), 1, gather=lambda s: s)
    ref = nf4lib.quantize_weight(w)
    torch.cuda.synchronize()
    assert torch.equal(st.packed, ref.packed) and torch.equal(st.absmax_q, ref.absmax_q)
    assert torch.equal(st.absmax2, ref.absmax2) and torch.equal(st.offset, ref.offset)


def test_empty_shard_writes_the_mean(nf4lib, cuda_device):
    c1 = torch.rand(3 * 256 + 5, device=cuda_device) * 0.1
    sums = nf4lib.nf4_dq_run_sums(c1)
    empty = torch.empty(0, dtype=torch.float32, device=cuda_device)
    _, _, off = nf4lib.nf4_double_quantize_sharded(empty, sums, c1.numel())
    _, _, ref = nf4lib.nf4_double_quantize(c1)
    torch.cuda.synchronize()
    assert torch.equal(off.view(torch.int32), ref.view(torch.int32))
