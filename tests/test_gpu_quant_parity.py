"""GPU parity: nf4_quantize, nf4_double_quantize and nf4_dequantize through the
C ABI against the CPU oracle, bit-exact (codes, packed bytes, absmax, 8-bit
scales, c2, mu, dequantized fp32 and bf16 values, signed zeros included)."""
import numpy as np
import pytest
import torch

import nf4_workloads as wl
from conftest import check_guards, guarded

pytestmark = pytest.mark.gpu


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def f32bits(a) -> np.ndarray:
    return np.ascontiguousarray(a, np.float32).view(np.uint32)


def oracle_input(w_cpu: torch.Tensor) -> np.ndarray:
    return u16(w_cpu).ravel() if w_cpu.dtype == torch.bfloat16 else w_cpu.contiguous().numpy().ravel()


def dq_guarded(q, c1: torch.Tensor, centre=True):
    """nf4_double_quantize into guarded outputs (and workspace); checks the
    guards and returns (codes, c2, mu or None)."""
    dev = c1.device
    nb = c1.numel()
    nd = -(-nb // 256)
    q8, c2 = guarded(nb, torch.uint8, dev), guarded(nd, torch.float32, dev)
    off = guarded(1, torch.float32, dev) if centre else None
    ws = guarded(q.nf4_double_quantize_workspace_size(nb), torch.uint8, dev)
    q.nf4_double_quantize(c1, centre=centre, absmax_q=q8, absmax2=c2, offset=off, workspace=ws)
    torch.cuda.synchronize()
    check_guards(q8, c2, off, ws)
    return q8, c2, off


def run_round_trip(q, oracle_mod, w_cpu: torch.Tensor, centre=True):
    dev = torch.device("cuda:0")
    w = w_cpu.to(dev)
    n = w.numel()
    nb = -(-n // 64)
    nd = -(-nb // 256)
    packed, absmax = guarded(n // 2, torch.uint8, dev), guarded(nb, torch.float32, dev)
    q.nf4_quantize(w.reshape(-1), packed=packed, absmax=absmax)
    q8, c2 = guarded(nb, torch.uint8, dev), guarded(nd, torch.float32, dev)
    off = guarded(1, torch.float32, dev) if centre else None
    ws = guarded(q.nf4_double_quantize_workspace_size(nb), torch.uint8, dev)
    q.nf4_double_quantize(absmax, centre=centre, absmax_q=q8, absmax2=c2, offset=off, workspace=ws)
    f32, b16 = guarded(n, torch.float32, dev), guarded(n, torch.bfloat16, dev)
    nodq = guarded(n, torch.float32, dev)
    q.nf4_dequantize(packed, q8, c2, off, n, torch.float32, out=f32)
    q.nf4_dequantize(packed, q8, c2, off, n, torch.bfloat16, out=b16)
    q.nf4_dequantize(packed, None, absmax, None, n, torch.float32, out=nodq)
    torch.cuda.synchronize()
    check_guards(packed, absmax, q8, c2, off, ws, f32, b16, nodq)

    op, oa = oracle_mod.quantize(oracle_input(w_cpu))
    assert np.array_equal(packed.cpu().numpy(), op), "packed codes differ"
    assert np.array_equal(f32bits(absmax.cpu().numpy()), f32bits(oa)), "absmax differs"
    oq8, oc2, omu = oracle_mod.double_quantize(oa, centre=centre)
    assert np.array_equal(q8.cpu().numpy(), oq8), "8-bit scale codes differ"
    assert np.array_equal(f32bits(c2.cpu().numpy()), f32bits(oc2)), "c2 differs"
    if centre:
        assert f32bits(off.cpu().numpy())[0] == f32bits([omu])[0], "mean differs"
    of = oracle_mod.dequantize(op, oq8, oc2, omu if centre else None, n, "f32")
    ob = oracle_mod.dequantize(op, oq8, oc2, omu if centre else None, n, "bf16")
    assert np.array_equal(f32bits(f32.cpu().numpy()), f32bits(of)), "fp32 dequant differs"
    assert np.array_equal(u16(b16), ob), "bf16 dequant differs"
    on = oracle_mod.dequantize(op, None, oa, None, n, "f32")
    assert np.array_equal(f32bits(nodq.cpu().numpy()), f32bits(on)), "no-DQ dequant differs"


def test_tiny_round_trip(nf4lib, oracle_mod, cuda_device):
    run_round_trip(nf4lib, oracle_mod, wl.weight_case(wl.TINY))


def test_projection_round_trip(nf4lib, oracle_mod, cuda_device):
    run_round_trip(nf4lib, oracle_mod, wl.weight_case(wl.PROJECTION))


def test_projection_without_centring(nf4lib, oracle_mod, cuda_device):
    run_round_trip(nf4lib, oracle_mod, wl.weight_case(wl.PROJECTION), centre=False)


@pytest.mark.parametrize("n", [2, 62, 64, 66, 130, 64 * 37 + 18, 16384 * 3 + 64 * 5 + 6])
def test_ragged_sizes(nf4lib, oracle_mod, cuda_device, n):
    w = wl.weight((n,), 0.02, 100 + n, "f32")
    run_round_trip(nf4lib, oracle_mod, w)
    run_round_trip(nf4lib, oracle_mod, w.to(torch.bfloat16))


def test_empty_input(nf4lib, cuda_device):
    w = torch.empty(0, device=cuda_device)
    packed, absmax = nf4lib.nf4_quantize(w)
    assert packed.numel() == 0 and absmax.numel() == 0


def tie_and_edge_tensor(oracle_mod) -> torch.Tensor:
    """Blocks built to hit exact ties, near-threshold quotients, zero and
    signed-zero elements, subnormal and huge scales."""
    q = oracle_mod.codebook().astype(np.float64)
    mids = (q[:-1] + q[1:]) / 2
    blocks = []
    # ties: c1 = 1, elements exactly at representable midpoints
    b = np.zeros(64, np.float32)
    b[0] = 1.0
    for i, m in enumerate(mids):
        b[1 + i] = np.float32(m)
        b[17 + i] = np.nextafter(np.float32(m), np.float32(2))
        b[33 + i] = np.nextafter(np.float32(m), np.float32(-2))
    b[48] = -0.0
    blocks.append(b)
    # the same with a non-power-of-two scale
    blocks.append((b * np.float32(0.0371)).astype(np.float32))
    # all zeros / negative zeros
    blocks.append(np.full(64, -0.0, np.float32))
    # subnormal-scale block and huge-scale block
    rng = np.random.default_rng(9)
    blocks.append((rng.standard_normal(64) * 1e-41).astype(np.float32))
    blocks.append((rng.standard_normal(64) * 1e37).astype(np.float32))
    blocks.append((rng.standard_normal(64) * 2.0 ** -126).astype(np.float32))
    # quotients a few ulps either side of every threshold, for several scales
    for c in (1.0, 0.7, 3.3e-3, 1.7e5):
        b = np.zeros(64, np.float32)
        b[0] = np.float32(c)
        k = 1
        for m in mids[:12]:
            t = np.float32(m * c)
            for d in (-2, 0, 2):
                v = t
                for _ in range(abs(d)):
                    v = np.nextafter(v, np.float32(np.sign(d) * np.inf))
                if k < 64:
                    b[k] = v
                    k += 1
        blocks.append(b)
    mixed = wl.random_bits_f32(64 * 40, 12).numpy()
    return torch.from_numpy(np.concatenate(blocks + [mixed]).astype(np.float32))


def test_ties_and_edge_values(nf4lib, oracle_mod, cuda_device):
    w = tie_and_edge_tensor(oracle_mod)
    dev = cuda_device
    n = w.numel()
    packed, absmax = guarded(n // 2, torch.uint8, dev), guarded(n // 64, torch.float32, dev)
    nf4lib.nf4_quantize(w.to(dev), packed=packed, absmax=absmax)
    op, oa = oracle_mod.quantize(w.numpy())
    assert np.array_equal(packed.cpu().numpy(), op)
    assert np.array_equal(f32bits(absmax.cpu().numpy()), f32bits(oa))
    # dequantize without DQ: exact including signed zeros
    out = guarded(n, torch.float32, dev)
    nf4lib.nf4_dequantize(packed, None, absmax, None, n, torch.float32, out=out)
    ref = oracle_mod.dequantize(op, None, oa, None, n, "f32")
    assert np.array_equal(f32bits(out.cpu().numpy()), f32bits(ref))
    check_guards(packed, absmax, out)


def test_dq_sequential_fallback_and_zero_runs(nf4lib, oracle_mod, cuda_device):
    """Runs whose constants span more than 2^21 in magnitude take the
    sequential fp64 sum; runs of equal constants give c2 = 0."""
    rng = np.random.default_rng(13)
    c1 = rng.uniform(0.01, 0.1, 256 * 70 + 17).astype(np.float32)
    c1[256 * 3: 256 * 4] = (rng.uniform(0, 1, 256) * 2.0 ** rng.integers(-60, 0, 256)).astype(np.float32)
    c1[256 * 5: 256 * 6] = np.float32(1e-40)
    c1[256 * 7] = np.float32(3e30)
    c1[256 * 9: 256 * 10] = 0.0
    dev = cuda_device
    for centre in (True, False):
        q8, c2, off = dq_guarded(nf4lib, torch.from_numpy(c1).to(dev), centre=centre)
        oq8, oc2, omu = oracle_mod.double_quantize(c1, centre=centre)
        assert np.array_equal(q8.cpu().numpy(), oq8)
        assert np.array_equal(f32bits(c2.cpu().numpy()), f32bits(oc2))
        if centre:
            assert f32bits(off.cpu().numpy())[0] == f32bits([omu])[0]
    # every constant equal to the mean: c2 = 0 and code 0
    c1 = np.full(1000, 0.0625, np.float32)
    q8, c2, off = dq_guarded(nf4lib, torch.from_numpy(c1).to(dev))
    assert float(off.item()) == 0.0625 and torch.all(c2 == 0) and torch.all(q8 == 0)


def test_many_chunks_mean(nf4lib, oracle_mod, cuda_device):
    """More than one chunk of 32 runs, ragged last chunk (tree across chunks)."""
    rng = np.random.default_rng(14)
    c1 = (rng.standard_normal(256 * 1000 + 100) ** 2 * 0.01).astype(np.float32)
    q8, c2, off = dq_guarded(nf4lib, torch.from_numpy(c1).to(cuda_device))
    oq8, oc2, omu = oracle_mod.double_quantize(c1)
    assert f32bits(off.cpu().numpy())[0] == f32bits([omu])[0]
    assert np.array_equal(q8.cpu().numpy(), oq8)
    assert np.array_equal(f32bits(c2.cpu().numpy()), f32bits(oc2))


def test_stream_ordering_on_side_stream(nf4lib, oracle_mod, cuda_device):
    w = wl.weight((512, 512), 0.02, 21, "bf16")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        wd = w.to(cuda_device, non_blocking=False)
        packed, absmax = nf4lib.nf4_quantize(wd.reshape(-1), stream=s)
        out = nf4lib.nf4_dequantize(packed, None, absmax, None, w.numel(), torch.bfloat16, stream=s)
    s.synchronize()
    op, oa = oracle_mod.quantize(u16(w).ravel())
    assert np.array_equal(packed.cpu().numpy(), op)
    assert np.array_equal(u16(out), oracle_mod.dequantize(op, None, oa, None, w.numel(), "bf16"))


def test_large_weight_dequant_element_by_element(nf4lib, oracle_mod, cuda_device):
    """The 14336 x 4096 training weight (58.7 M elements, above 2^25, so the
    dequantizer's large-output launch shape): codes, constants and every
    element of the bf16 and fp32 dequantization against the oracle."""
    w = wl.weight((14336, 4096), 0.02, wl.GEMM_TRAIN.seed, "bf16")
    n = w.numel()
    dev = cuda_device
    st = nf4lib.quantize_weight(w.to(dev))
    op, oa = oracle_mod.quantize(u16(w).ravel())
    oq8, oc2, omu = oracle_mod.double_quantize(oa)
    assert np.array_equal(st.packed.cpu().numpy(), op)
    assert np.array_equal(st.absmax_q.cpu().numpy(), oq8)
    assert np.array_equal(f32bits(st.absmax2.cpu().numpy()), f32bits(oc2))
    assert f32bits(st.offset.cpu().numpy())[0] == f32bits([omu])[0]
    for dt, name in ((torch.bfloat16, "bf16"), (torch.float32, "f32")):
        out = guarded(n, dt, dev)
        nf4lib.nf4_dequantize(st.packed, st.absmax_q, st.absmax2, st.offset, n, dt, out=out)
        torch.cuda.synchronize()
        check_guards(out)
        ref = oracle_mod.dequantize(op, oq8, oc2, omu, n, name)
        got = u16(out) if name == "bf16" else f32bits(out.cpu().numpy())
        exp = ref if name == "bf16" else f32bits(ref)
        bad = np.flatnonzero(got != exp)
        assert bad.size == 0, f"{name}: {bad.size} elements differ, first at {bad[:5]}"
        del out


def test_70b_mlp_weight_dequant_sampled_runs(nf4lib, oracle_mod, cuda_device):
    """The 28672 x 8192 MLP weight (234.9 M elements): codes, constants and
    mean in full; the bf16 dequantization element by element on 48 whole
    runs of 16,384 elements (one second-level block each) spread over the
    tensor, first and last run included."""
    w = wl.weight((28672, 8192), 0.02, wl.GEMM_70B_MLP.seed, "bf16")
    n = w.numel()
    run = 64 * 256
    dev = cuda_device
    st = nf4lib.quantize_weight(w.to(dev))
    out = guarded(n, torch.bfloat16, dev)
    nf4lib.nf4_dequantize(st.packed, st.absmax_q, st.absmax2, st.offset, n, torch.bfloat16, out=out)
    torch.cuda.synchronize()
    check_guards(out)
    bits = u16(w).ravel()
    del w
    op, oa = oracle_mod.quantize(bits)
    oq8, oc2, omu = oracle_mod.double_quantize(oa)
    assert np.array_equal(st.packed.cpu().numpy(), op)
    assert np.array_equal(st.absmax_q.cpu().numpy(), oq8)
    assert np.array_equal(f32bits(st.absmax2.cpu().numpy()), f32bits(oc2))
    assert f32bits(st.offset.cpu().numpy())[0] == f32bits([omu])[0]
    runs = n // run
    rng = np.random.default_rng(70)
    pick = np.unique(np.concatenate([[0, runs - 1], rng.choice(runs, 46, replace=False)]))
    for d in pick:
        e0, e1 = d * run, (d + 1) * run
        ref = oracle_mod.dequantize(op[e0 // 2:e1 // 2], oq8[e0 // 64:e1 // 64], oc2[d:d + 1], omu, run, "bf16")
        assert np.array_equal(u16(out[e0:e1]), ref), f"run {d} differs"


def wide_range_weight(n, seed):
    """Gaussian weights whose 64-blocks are scaled by 2^U, U uniform in
    [-40, 8]: the block constants of a run span far more than 2^21, so the
    fp64 run sums of the centring mean take the sequential order."""
    g = torch.Generator().manual_seed(seed)
    w = torch.randn(n, generator=g)
    nb = -(-n // 64)
    e = torch.randint(-40, 9, (nb,), generator=g).to(torch.float32)
    return (w * torch.pow(2.0, e).repeat_interleave(64)[:n]).contiguous()


@pytest.mark.parametrize("n,dtype,centre", [(4096 * 4096, "bf16", True), (14336 * 4096, "bf16", True),
                                            (16384 * 3 + 64 * 5 + 6, "f32", True), (2, "bf16", True),
                                            (16384 * 2100 + 130, "bf16", True), (256 * 512, "f32", False),
                                            (16384 * 7 + 4, "wide", True)])
def test_quantize_dq_one_call(nf4lib, oracle_mod, cuda_device, n, dtype, centre):
    """nf4_quantize_dq (quantizer writing the run sums, then one double
    quantization kernel; above 2048 runs a chunk-sum kernel too) against the
    oracle's quantize + double quantize, bit for bit, outputs and workspace
    guarded."""
    if dtype == "wide":
        w_cpu = wide_range_weight(n, 5)
    else:
        w_cpu = wl.weight((n,), 0.02, 40 + n % 1000, "f32", outliers=True)
        if dtype == "bf16":
            w_cpu = w_cpu.to(torch.bfloat16)
    dev = cuda_device
    nb = -(-n // 64)
    nd = -(-nb // 256)
    packed, q8 = guarded(n // 2, torch.uint8, dev), guarded(nb, torch.uint8, dev)
    c2 = guarded(nd, torch.float32, dev)
    off = guarded(1, torch.float32, dev) if centre else None
    ws = guarded(nf4lib.nf4_quantize_dq_workspace_size(n), torch.uint8, dev)
    nf4lib.nf4_quantize_dq(w_cpu.to(dev), centre=centre, packed=packed, absmax_q=q8, absmax2=c2, offset=off,
                           workspace=ws)
    nf4lib.nf4_device_status()
    check_guards(packed, q8, c2, off, ws)
    op, oa = oracle_mod.quantize(oracle_input(w_cpu))
    oq8, oc2, omu = oracle_mod.double_quantize(oa, centre=centre)
    assert np.array_equal(packed.cpu().numpy(), op)
    assert np.array_equal(q8.cpu().numpy(), oq8)
    assert np.array_equal(f32bits(c2.cpu().numpy()), f32bits(oc2))
    if centre:
        assert f32bits(off.cpu().numpy())[0] == f32bits([omu])[0]
    # the fp32 constants passed through the workspace (its first nb words)
    assert np.array_equal(f32bits(ws[:4 * nb].view(torch.float32).cpu().numpy()), f32bits(oa))


def test_quantize_wide_range_constants(nf4lib, oracle_mod, cuda_device):
    """nf4_quantize and nf4_double_quantize on block constants spanning
    2^-40 .. 2^8 (sequential fp64 order for the mean)."""
    run_round_trip(nf4lib, oracle_mod, wide_range_weight(16384 * 5 + 64 * 9 + 2, 6))
