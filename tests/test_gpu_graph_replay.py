"""The benchmark times each call as CUDA-graph replays of back-to-back
launches (programmatic dependent launch between them).  These tests check
that such replays compute exactly what the same calls compute when launched
one by one: quantize + double quantize, dequantize, and the fused linear on
its three paths (decode kernel with one and two token tiles, 256-token GEMM),
each replayed with inputs rotating over several copies, outputs compared bit
for bit with the eager calls (and the eager calls are the ones the parity
tests check against the oracle)."""
import pytest
import torch

import nf4_workloads as wl

pytestmark = pytest.mark.gpu


def replay(fns):
    """Capture every fn of `fns` in one graph, in order, and replay it twice."""
    for f in fns:  # first calls outside the capture (one-time set-up)
        f()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for f in fns:
            f()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    del g


def test_quantize_and_dequantize_replayed(nf4lib, cuda_device):
    dev = cuda_device
    C = 3
    ws = [wl.weight((1024, 2048), 0.02, 70 + k, "bf16", outliers=True).to(dev).reshape(-1) for k in range(C)]
    n = ws[0].numel()
    nb = n // 64
    eager = [nf4lib.nf4_quantize_dq(w) for w in ws]
    deq_eager = [nf4lib.nf4_dequantize(p, q8, c2, off, n, torch.bfloat16) for p, q8, c2, off in eager]
    outs = [(torch.empty(n // 2, dtype=torch.uint8, device=dev), torch.empty(nb, dtype=torch.uint8, device=dev),
             torch.empty(nb // 256, device=dev), torch.empty(1, device=dev)) for _ in range(C)]
    wsp = torch.empty(nf4lib.nf4_quantize_dq_workspace_size(n), dtype=torch.uint8, device=dev)
    deq = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(C)]

    def qdq(k):
        nf4lib.nf4_quantize_dq(ws[k], packed=outs[k][0], absmax_q=outs[k][1], absmax2=outs[k][2],
                               offset=outs[k][3], workspace=wsp)
        nf4lib.nf4_dequantize(*outs[k], n, torch.bfloat16, out=deq[k])
    replay([lambda k=k: qdq(k) for k in range(C)])
    for k in range(C):
        for a, b in zip(outs[k], eager[k]):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
        assert torch.equal(deq[k], deq_eager[k])


@pytest.mark.parametrize("M,K,N,r", [(1, 4096, 2048, 16), (16, 2048, 4096, 16), (512, 1024, 1024, 64)])
def test_linear_replayed(nf4lib, cuda_device, M, K, N, r):
    dev = cuda_device
    C = 3
    c = wl.LinearCase("graph", M, K, N, r, 0.5, 90 + M)
    W, x, A, B = wl.linear_inputs(c)
    st = nf4lib.quantize_weight(W.to(dev))
    g = torch.Generator().manual_seed(M)
    xs = [torch.randn(M, K, generator=g).to(torch.bfloat16).to(dev) for _ in range(C)]
    Ad, Bd = A.to(dev), B.to(dev)
    eager = [nf4lib.nf4_lora_linear_fwd(xk, st.packed, st.absmax_q, st.absmax2, st.offset, N, Ad, Bd, c.scaling)
             for xk in xs]
    ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for _ in range(C)]
    wsp = torch.empty(max(16, nf4lib.nf4_lora_linear_workspace_size(M, r)), dtype=torch.uint8, device=dev)
    replay([lambda k=k: nf4lib.nf4_lora_linear_fwd(xs[k], st.packed, st.absmax_q, st.absmax2, st.offset, N, Ad, Bd,
                                                   c.scaling, y=ys[k], workspace=wsp) for k in range(C)])
    assert nf4lib.nf4_device_status() == 0
    for k in range(C):
        assert torch.equal(ys[k], eager[k]), k
