"""GPU parity of nf4_lora_linear_fwd (the fused frozen-base LoRA linear)
through the C ABI against the CPU oracle (fp64), within the matmul tolerance:
max relative error <= 1e-2 and mean relative error < 2e-3, the denominator
floored at 1e-2 of the reference's rms.  Special cases reduce to library
routines: with no LoRA term the result equals torch.matmul on the bf16 output
of nf4_dequantize."""
import numpy as np
import pytest
import torch

import nf4_workloads as wl
from conftest import MATMUL_MAX_REL, MATMUL_MEAN_REL, check_guards, guarded, rel_error_stats

pytestmark = pytest.mark.gpu


def u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def quantize_on_gpu(q, W: torch.Tensor, dev, dq=True):
    return q.quantize_weight(W.to(dev), double_quant=dq)


def linear(q, x, st, N, A=None, B=None, s=1.0, ws_bytes=None):
    """nf4_lora_linear_fwd with its output and workspace between poisoned
    guard regions (checked after the call); ws_bytes overrides the
    workspace size the call is given."""
    M = x.shape[0]
    r = 0 if A is None else A.shape[0]
    dev = x.device
    y = guarded((M, N), torch.bfloat16, dev)
    if ws_bytes is None:
        ws_bytes = q.nf4_lora_linear_workspace_size(M, r)
    ws = guarded(ws_bytes, torch.uint8, dev) if ws_bytes > 0 else None
    q.nf4_lora_linear_fwd(x, st.packed, st.absmax_q, st.absmax2, st.offset, N, A, B, s, y=y, workspace=ws)
    q.nf4_device_status()
    check_guards(y, ws)
    return y


def oracle_linear(oracle_mod, st, x, A, B, r, s, rows=None):
    K = x.shape[1]
    N = st.shape[0]
    packed = st.packed.cpu().numpy()
    scales = st.absmax2.cpu().numpy()
    q8 = None if st.absmax_q is None else st.absmax_q.cpu().numpy()
    mu = None if st.offset is None else np.float32(st.offset.cpu().numpy()[0])
    return oracle_mod.lora_linear(u16(x), K, N, packed, q8, scales, mu,
                                  None if A is None else u16(A), None if B is None else u16(B), r, s, rows=rows)


def check(y: torch.Tensor, ref: np.ndarray):
    mx, mean, fro = rel_error_stats(y.float().cpu().numpy(), ref)
    assert mx <= MATMUL_MAX_REL and mean < MATMUL_MEAN_REL, (mx, mean, fro)
    return mx, mean, fro


@pytest.mark.parametrize("case", wl.GEMV_CASES, ids=lambda c: f"T{c.M}")
def test_decode_gemv_full_size(nf4lib, oracle_mod, cuda_device, case):
    W, x, A, B = wl.linear_inputs(case)
    st = quantize_on_gpu(nf4lib, W, cuda_device)
    y = linear(nf4lib, x.to(cuda_device), st, case.N, A.to(cuda_device), B.to(cuda_device), case.scaling)
    torch.cuda.synchronize()
    check(y, oracle_linear(oracle_mod, st, x, A, B, case.r, case.scaling))


@pytest.mark.parametrize("M,K,N,r,dq", [(1, 192, 200, 16, True), (7, 64, 40, 32, True), (16, 320, 96, 64, False),
                                        (9, 1024, 8, 16, True), (16, 4096, 1000, 0, True),
                                        (3, 256, 24, 64, False), (5, 768, 4000, 32, True),
                                        (12, 512, 2400, 16, False), (8, 8192, 520, 64, True)])
def test_gemv_ragged_shapes(nf4lib, oracle_mod, cuda_device, M, K, N, r, dq):
    c = wl.LinearCase("ragged", M, K, N, r, 1.5, 31 + M + K + N)
    W, x, A, B = wl.linear_inputs(c, with_lora=r > 0)
    st = quantize_on_gpu(nf4lib, W, cuda_device, dq)
    dA = None if A is None else A.to(cuda_device)
    dB = None if B is None else B.to(cuda_device)
    y = linear(nf4lib, x.to(cuda_device), st, N, dA, dB, c.scaling)
    torch.cuda.synchronize()
    check(y, oracle_linear(oracle_mod, st, x, A, B, r, c.scaling))


@pytest.mark.parametrize("M,K,N,r,dq", [(3, 5120, 264, 16, True),    # 20 slices of 256 columns: warps take several
                                        (8, 1024, 4000, 0, True),     # 4 slices: four warp groups split the tiles
                                        (2, 64, 136, 32, False),      # one slice: sixteen groups
                                        (6, 1344, 48, 64, True),      # ragged last slice (21 blocks)
                                        (1, 4096, 33024, 16, True),   # more tiles per CTA than shared memory holds
                                        (5, 128, 8, 16, True),        # one partial tile
                                        # two token tiles (9..16 tokens), slices of 128 columns
                                        (11, 5120, 264, 16, True),    # 40 slices: warps take two or three
                                        (13, 11008, 520, 16, True),   # 86 slices, several tiles per CTA
                                        (16, 1024, 4000, 0, True),    # 8 slices: two warp groups
                                        (9, 64, 136, 32, False),      # one slice, its second block outside K
                                        (12, 192, 40, 16, True),      # odd block count: half of the last slice
                                        (14, 1344, 48, 64, True),     # ragged last slice (21 blocks)
                                        (16, 4096, 33024, 16, True),  # chunks that use both partial regions
                                        (10, 128, 8, 16, True)])      # one partial tile
def test_decode_work_splits(nf4lib, oracle_mod, cuda_device, M, K, N, r, dq):
    """The decode kernel (up to 16 tokens, in one or two tiles of 8) splits K
    into slices of 256 or 128 columns over the warps of a CTA and keeps
    per-slice partial tiles in shared memory; these shapes reach each way of
    splitting."""
    c = wl.LinearCase("decode split", M, K, N, r, 0.5, 977 + M + K + N)
    W, x, A, B = wl.linear_inputs(c, with_lora=r > 0)
    st = quantize_on_gpu(nf4lib, W, cuda_device, dq)
    dA = None if A is None else A.to(cuda_device)
    dB = None if B is None else B.to(cuda_device)
    y = linear(nf4lib, x.to(cuda_device), st, N, dA, dB, c.scaling)
    torch.cuda.synchronize()
    check(y, oracle_linear(oracle_mod, st, x, A, B, r, c.scaling))


@pytest.mark.parametrize("M,K,N,r", [(1, 512, 2400, 16), (13, 256, 200, 64), (4, 192, 64, 32), (40, 512, 264, 16)])
def test_linear_double_quant_without_centring(nf4lib, oracle_mod, cuda_device, M, K, N, r):
    """Block constants decoded as E4M3 * c2 (no centring offset), through
    the decode kernel (one and two token tiles) and the tensor-core GEMM."""
    c = wl.LinearCase("no centring", M, K, N, r, 1.25, 211 + M + K + N)
    W, x, A, B = wl.linear_inputs(c)
    st = nf4lib.quantize_weight(W.to(cuda_device), centre=False)
    assert st.offset is None
    y = linear(nf4lib, x.to(cuda_device), st, N, A.to(cuda_device), B.to(cuda_device), c.scaling)
    torch.cuda.synchronize()
    check(y, oracle_linear(oracle_mod, st, x, A, B, r, c.scaling))


def test_gemv_without_lora_equals_matmul_on_dequantized(nf4lib, cuda_device):
    c = wl.GEMV_CASES[2]
    W, x, _, _ = wl.linear_inputs(c, with_lora=False)
    st = quantize_on_gpu(nf4lib, W, cuda_device)
    xd = x.to(cuda_device)
    y = linear(nf4lib, xd, st, c.N)
    wb = nf4lib.nf4_dequantize(st.packed, st.absmax_q, st.absmax2, st.offset, c.N * c.K).view(c.N, c.K)
    ref = torch.matmul(xd.float(), wb.float().t())
    torch.cuda.synchronize()
    check(y, ref.cpu().numpy())


# ---------------------------------------------------------------- tensor-core GEMM (M > 16)
@pytest.mark.parametrize("M,K,N,r,dq", [(17, 64, 8, 0, True), (100, 192, 136, 16, True), (256, 256, 128, 64, True),
                                        (300, 320, 264, 32, False), (513, 128, 256, 16, True),
                                        # 13 and 7 pipeline steps: the stage ring wraps, ragged last round
                                        (70, 768, 72, 32, True), (140, 448, 264, 0, False)])
def test_gemm_small_shapes_full_output(nf4lib, oracle_mod, cuda_device, M, K, N, r, dq):
    c = wl.LinearCase("gemm small", M, K, N, r, 0.75, 57 + M + K + N)
    W, x, A, B = wl.linear_inputs(c, with_lora=r > 0)
    st = quantize_on_gpu(nf4lib, W, cuda_device, dq)
    dA = None if A is None else A.to(cuda_device)
    dB = None if B is None else B.to(cuda_device)
    y = linear(nf4lib, x.to(cuda_device), st, N, dA, dB, c.scaling)
    nf4lib.nf4_device_status()
    check(y, oracle_linear(oracle_mod, st, x, A, B, r, c.scaling))


def sampled_rows(M, count, seed):
    rng = np.random.default_rng(seed)
    rows = np.sort(rng.choice(M, size=min(count, M), replace=False)).astype(np.int64)
    return np.unique(np.concatenate([rows, [0, M - 1]])).astype(np.int64)


@pytest.mark.parametrize("case,nrows", [(wl.GEMM_TRAIN, 192), (wl.GEMM_70B_MLP, 48), (wl.GEMM_DOWN_PROJ, 64),
                                        (wl.GEMM_K_PROJ, 128)],
                         ids=["train4096", "mlp70b", "down_proj", "k_proj"])
def test_gemm_full_size_sampled_rows(nf4lib, oracle_mod, cuda_device, case, nrows):
    W, x, A, B = wl.linear_inputs(case)
    st = quantize_on_gpu(nf4lib, W, cuda_device)
    del W
    y = linear(nf4lib, x.to(cuda_device), st, case.N, A.to(cuda_device), B.to(cuda_device), case.scaling)
    nf4lib.nf4_device_status()
    rows = sampled_rows(case.M, nrows, case.seed)
    ref = oracle_linear(oracle_mod, st, x, A, B, case.r, case.scaling, rows=rows)
    check(y[torch.from_numpy(rows).to(cuda_device)], ref)


def test_gemm_partial_last_wave(nf4lib, oracle_mod, cuda_device):
    """150 tiles of 128 x 256 on 148 SMs (a second, nearly empty wave); the
    sampled rows include the last 8 tokens, which meet the last tiles."""
    c = wl.LinearCase("gemm partial wave", 512, 1024, 9600, 16, 0.5, 4242)
    W, x, A, B = wl.linear_inputs(c)
    st = quantize_on_gpu(nf4lib, W, cuda_device)
    y = linear(nf4lib, x.to(cuda_device), st, c.N, A.to(cuda_device), B.to(cuda_device), c.scaling)
    nf4lib.nf4_device_status()
    rows = np.unique(np.concatenate([sampled_rows(c.M, 8, c.seed), np.arange(c.M - 8, c.M)])).astype(np.int64)
    ref = oracle_linear(oracle_mod, st, x, A, B, c.r, c.scaling, rows=rows)
    check(y[torch.from_numpy(rows).to(cuda_device)], ref)


def test_gemm_without_lora_equals_matmul_on_dequantized(nf4lib, cuda_device):
    c = wl.LinearCase("gemm vs torch", 1024, 2048, 3072, 0, 1.0, 77)
    W, x, _, _ = wl.linear_inputs(c, with_lora=False)
    st = quantize_on_gpu(nf4lib, W, cuda_device)
    xd = x.to(cuda_device)
    y = linear(nf4lib, xd, st, c.N)
    wb = nf4lib.nf4_dequantize(st.packed, st.absmax_q, st.absmax2, st.offset, c.N * c.K).view(c.N, c.K)
    ref = torch.matmul(xd.float(), wb.float().t())
    nf4lib.nf4_device_status()
    check(y, ref.cpu().numpy())


def test_gemm_and_gemv_agree_on_shared_rows(nf4lib, cuda_device):
    """T = 16 through the GEMV path equals the first 16 rows of a 64-row GEMM."""
    c = wl.LinearCase("agree", 64, 1024, 512, 16, 2.0, 91)
    W, x, A, B = wl.linear_inputs(c)
    st = quantize_on_gpu(nf4lib, W, cuda_device)
    xd, Ad, Bd = x.to(cuda_device), A.to(cuda_device), B.to(cuda_device)
    y64 = linear(nf4lib, xd, st, c.N, Ad, Bd, c.scaling)
    y16 = linear(nf4lib, xd[:16].contiguous(), st, c.N, Ad, Bd, c.scaling)
    nf4lib.nf4_device_status()
    check(y16, y64[:16].float().cpu().numpy())


@pytest.mark.parametrize("M,K,N,r,dq", [(9, 1024, 8, 16, True), (12, 512, 2400, 16, False), (16, 512, 2400, 64, True),
                                        (16, 2048, 640, 32, True), (11, 8192, 1000, 0, True),
                                        (16, 64, 18936, 32, True), (10, 4096, 11008, 0, True)])
def test_two_token_tiles_repeatable(nf4lib, oracle_mod, cuda_device, M, K, N, r, dq):
    """9 to 16 tokens (the decode kernel's two 8-token tiles): the result
    matches the oracle and is bitwise the same on every run and with a
    workspace larger than required (partial tiles are added in slot order,
    never in arrival order).  Shapes cover one partial row tile, no adapter,
    more row tiles than SMs, and K of one block."""
    c = wl.LinearCase("two tiles", M, K, N, r, 1.25, 57 + M + K + N)
    W, x, A, B = wl.linear_inputs(c, with_lora=r > 0)
    st = quantize_on_gpu(nf4lib, W, cuda_device, dq)
    xd = x.to(cuda_device)
    dA = None if A is None else A.to(cuda_device)
    dB = None if B is None else B.to(cuda_device)
    ref = oracle_linear(oracle_mod, st, x, A, B, r, c.scaling)
    need = nf4lib.nf4_lora_linear_workspace_size(M, r)
    assert need == (M * ((2 * r + 63) // 64) * 64 * 2 if r > 0 else 0)
    outs = []
    for ws_bytes in (need, need, need + 4096, need):
        outs.append(linear(nf4lib, xd, st, N, dA, dB, c.scaling, ws_bytes=ws_bytes))
    torch.cuda.synchronize()
    assert nf4lib.nf4_device_status() == 0
    for y in outs:
        check(y, ref)
    assert all(torch.equal(outs[0], y) for y in outs[1:])


def test_two_token_tiles_back_to_back(nf4lib, cuda_device):
    """16-token decode calls queued back to back on one stream (programmatic
    dependent launch between them), with and without an adapter, reuse one
    workspace: every output equals the same call run alone, and no call
    writes outside its output or the shared workspace."""
    c = wl.LinearCase("decode b2b", 16, 2048, 4096, 16, 2.0, 93)
    W, x, A, B = wl.linear_inputs(c)
    st = quantize_on_gpu(nf4lib, W, cuda_device)
    xd, Ad, Bd = x.to(cuda_device), A.to(cuda_device), B.to(cuda_device)
    alone = [linear(nf4lib, xd, st, c.N, a, b, c.scaling) for a, b in ((Ad, Bd), (None, None))]
    ws = guarded(nf4lib.nf4_lora_linear_workspace_size(16, 16), torch.uint8, cuda_device)
    ys = []
    for i in range(12):
        a, b = ((Ad, Bd), (None, None))[i % 2]
        y = guarded((c.M, c.N), torch.bfloat16, cuda_device)
        nf4lib.nf4_lora_linear_fwd(xd, st.packed, st.absmax_q, st.absmax2, st.offset, c.N, a, b, c.scaling, y=y,
                                   workspace=ws)
        ys.append(y)
    torch.cuda.synchronize()
    assert nf4lib.nf4_device_status() == 0
    check_guards(ws, *ys)
    for i, y in enumerate(ys):
        assert torch.equal(y, alone[i % 2]), i
