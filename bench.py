"""Benchmark of the NF4 hot path on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass over every call of the path on per-GPU synthetic inputs
(the configurations: tiny round trip = parity only; the rest timed here):
  - projection 4096x4096 bf16 (0.1% x10 outliers): nf4_quantize,
    nf4_double_quantize, both together, nf4_dequantize to bf16 (the headline
    value: NF4 dequant GB/s), to fp32, and to bf16 from fp32 constants (no
    double quantization);
  - decode GEMV, nf4_lora_linear_fwd with x[T, 4096], T = 1, 4, 16, W
    11008x4096, r = 16, s = 2;
  - training GEMM, x[4096, 4096], W 14336x4096, r = 64, s = 0.25 (the kernel
    that dominates the step: the `roofline` object);
  - 70B MLP GEMM, x[2048, 8192], W 28672x8192, r = 16, s = 2;
  - one 8B-shaped decoder layer's seven weights: quantize + double-quantize +
    dequantize (the whole-model sweep is 32 such layers);
  - the same layer's seven linears at M = 4096 tokens, r = 64, through the
    fused NF4 path, and as unquantized bf16 LoRA GEMMs on cuBLAS (the
    comparison behind `overhead_vs_bf16_lora`; not this library's kernels);
  - backward (dx, dA, dB) and merge + requantize of the training GEMM.
Each call is captured R times back to back in a CUDA graph, its inputs
rotating over copies larger than the 126 MB L2 (no call reads a warm input),
and each graph replay is bracketed by CUDA events on the launching stream:
a call's time is its replays' time / R.  Inputs are resident in HBM before
timing.  `e2e` times nf4_dequantize through pinned host buffers.

With N > 1 (torchrun) every rank runs the same per-GPU workload on its own
data, plus one tensor sharded over the ranks (its runs' fp64 sums
all-gathered over NCCL for the double quantization's mean); times are the
maximum over ranks (weak scaling).  --impl reference times the CPU oracle on
rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NF4 dequant GB/s; fused NF4+LoRA linear TFLOP/s; % of HBM/tensor roofline"
BLOCK, DQ_BLOCK = 64, 256
BYTES_PER_PARAM_DQ = 0.5 + 1 / 64 + 4 / 16384
WORKLOAD = ("every call of the path, each replayed back to back: projection 4096x4096 bf16 (0.1% x10 outliers) "
            "quantize, double-quantize, quantize+DQ, dequantize to bf16 (headline value) / fp32 / bf16 without DQ; "
            "decode GEMV x[T,4096] T=1,4,16, W 11008x4096 r=16; training GEMM x[4096,4096] W 14336x4096 r=64; "
            "70B MLP GEMM x[2048,8192] W 28672x8192 r=16; one 8B-shaped layer's 7 weights quantize+DQ+dequantize "
            "and its 7 linears at M=4096 r=64 (vs bf16 LoRA on cuBLAS); backward and merge+requantize of the "
            "training GEMM")


# ------------------------------------------------------------------ algorithmic work per call
def quantize_bytes(n):   # read bf16 weight, write codes and fp32 absmax
    return n * 2 + n // 2 + (n // BLOCK) * 4


def dq_bytes(nb):        # read fp32 constants, write 8-bit codes, c2 and the mean
    return nb * 4 + nb + -(-nb // DQ_BLOCK) * 4 + 4


def quantize_dq_bytes(n):  # read the bf16 weight, write the stored format (codes, 8-bit constants, c2, mean)
    nb = -(-n // BLOCK)
    return n * 2 + n // 2 + nb + -(-nb // DQ_BLOCK) * 4 + 4


def dequant_bytes(n, out_bytes=2):  # read the quantized state once, write the weight
    nb = -(-n // BLOCK)
    return n // 2 + nb + -(-nb // DQ_BLOCK) * 4 + 4 + n * out_bytes


def linear_bytes(M, K, N, r):
    n = N * K
    nb = n // BLOCK
    return n // 2 + nb + -(-nb // DQ_BLOCK) * 4 + 4 + M * K * 2 + r * K * 2 + N * r * 2 + M * N * 2


def linear_flops(M, K, N, r):
    return 2 * M * N * K + 2 * M * r * (K + N)


# ------------------------------------------------------------------ distributed plumbing
def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(world, backend):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def reduce_max(values, world, device=None):
    """Element-wise maximum of a list of floats over all ranks."""
    import torch
    if world == 1:
        return list(values)
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def rank_seed(base, rank):
    """Each rank draws its own independent problem."""
    return base + 100_003 * rank


# ------------------------------------------------------------------ clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"nf4_bench_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "20"], stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
            return
        # the sampler takes a moment to start: the timed region begins once it
        # has written its first sample (or after 3 s)
        t0 = time.time()
        while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.02)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        self.proc.wait()
        rows = []
        with open(self.path) as f:
            for line in f:
                p = [x.strip() for x in line.split(",")]
                if len(p) >= 9:
                    rows.append(p)
        os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * (max(mx) if mx else 1)] or sm
        return {"sm_mhz": float(np.median(loaded)) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def code_digest(kernel_file):
    """First 16 hex digits of a sha256 over the kernel's source file and the
    local headers it includes (recursively, in include order), each with its
    comments removed and its white space collapsed: an edit to comments
    keeps a recorded capture valid, any change to the code voids it."""
    csrc = os.path.join(ROOT, "qlora_nf4_quantize_b200", "csrc")
    order, seen = [], set()

    def visit(name):
        if name in seen:
            return
        seen.add(name)
        order.append(name)
        with open(os.path.join(csrc, name)) as f:
            text = f.read()
        for inc in re.findall(r'#include\s+"([^"/]+)"', text):
            if os.path.exists(os.path.join(csrc, inc)):
                visit(inc)

    visit(kernel_file)
    h = hashlib.sha256()
    for name in order:
        with open(os.path.join(csrc, name)) as f:
            src = f.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(name.encode() + b"\0" + " ".join(src.split()).encode() + b"\0")
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current code of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        e = rec.get(kernel_file)
        if e and e.get("code_sha256_16") == code_digest(kernel_file):
            return e.get("dram_bytes_per_launch")
    except (OSError, ValueError):
        pass
    return None


# ------------------------------------------------------------------ our arm
class Segment:
    """One call of the path, replayed `reps` times back to back from a CUDA
    graph with its inputs rotating over copies (call j uses copy j mod C)."""

    def __init__(self, name, fns, reps, work, unit, launches, config):
        self.name, self.fns, self.reps, self.work, self.unit = name, fns, reps, work, unit
        self.launches, self.config = launches, config
        self.graph = None
        self.ms = 0.0

    def capture(self):
        import torch
        for f in self.fns:  # first calls outside the capture (one-time set-up)
            f()
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            for j in range(self.reps):
                self.fns[j % len(self.fns)]()
        torch.cuda.synchronize()


def build_segments(q, wl, dev, rank, world):
    """Every call the workloads name, with inputs resident in HBM.  Returns
    (segments, the projection weight on the CPU, handles kept for e2e)."""
    import torch
    segs = []
    wp, state = _projection_segments(q, wl, dev, rank, segs)
    _gemv_segments(q, wl, dev, rank, segs)
    for c, tag in ((wl.GEMM_TRAIN, "gemm_M4096"), (wl.GEMM_70B_MLP, "gemm_70B_M2048")):
        _gemm_segment(q, wl, dev, rank, segs, c, tag)
    _sweep_segment(q, wl, dev, segs)
    _layer_linear_segments(q, wl, dev, rank, segs)
    _bwd_merge_segments(q, wl, dev, rank, segs)
    torch.cuda.synchronize()
    return segs, wp, state


def _projection_segments(q, wl, dev, rank, segs):
    """Config 2: the projection 4096 x 4096 bf16 with outliers."""
    import torch
    wp = wl.weight((4096, 4096), 0.02, rank_seed(wl.PROJECTION["seed"], rank), "bf16", outliers=True)
    n = wp.numel()
    nb, nd = n // BLOCK, -(-(n // BLOCK) // DQ_BLOCK)
    C = 8
    W2 = [wp.to(dev).reshape(-1) for _ in range(C)]
    pk = [torch.empty(n // 2, dtype=torch.uint8, device=dev) for _ in range(C)]
    ab = [torch.empty(nb, dtype=torch.float32, device=dev) for _ in range(C)]
    q8 = [torch.empty(nb, dtype=torch.uint8, device=dev) for _ in range(C)]
    c2 = [torch.empty(nd, dtype=torch.float32, device=dev) for _ in range(C)]
    mu = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(C)]
    dq_ws = torch.empty(q.nf4_double_quantize_workspace_size(nb), dtype=torch.uint8, device=dev)
    deq = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(C)]
    deq32 = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(C)]
    for k in range(C):  # the quantized state every dequantize call reads
        q.nf4_quantize(W2[k], packed=pk[k], absmax=ab[k])
        q.nf4_double_quantize(ab[k], absmax_q=q8[k], absmax2=c2[k], offset=mu[k], workspace=dq_ws)
    # the double quantization alone rotates over 128 copies of the constants
    # (128 x 1.3 MB of inputs and outputs, more than the L2), so every call
    # reads its input from HBM
    CD = 128
    abx = [ab[k % C].clone() for k in range(CD)]
    q8x = [torch.empty(nb, dtype=torch.uint8, device=dev) for _ in range(CD)]
    c2x = [torch.empty(nd, dtype=torch.float32, device=dev) for _ in range(CD)]
    mux = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(CD)]
    ab_nodq = [a.clone() for a in ab]

    proj = "projection 4096x4096 bf16, 0.1% x10 outliers"
    segs.append(Segment("quantize", [lambda k=k: q.nf4_quantize(W2[k], packed=pk[k], absmax=ab_nodq[k])
                                     for k in range(C)], 16, quantize_bytes(n), "GB/s", 1, proj))
    segs.append(Segment("double_quantize", [lambda k=k: q.nf4_double_quantize(
        abx[k], absmax_q=q8x[k], absmax2=c2x[k], offset=mux[k], workspace=dq_ws) for k in range(CD)], CD,
        dq_bytes(nb), "GB/s", 2, f"{nb} block constants of the {proj}"))

    qdq_ws = torch.empty(q.nf4_quantize_dq_workspace_size(n), dtype=torch.uint8, device=dev)

    def f_qdq(k):  # the stored format in one call (its fp32 constants stay in the workspace)
        q.nf4_quantize_dq(W2[k], packed=pk[k], absmax_q=q8x[k], absmax2=c2x[k], offset=mux[k], workspace=qdq_ws)
    # launches: quantize, run sums, double quantization (1024 runs: no chunk sums)
    segs.append(Segment("quantize+dq", [lambda k=k: f_qdq(k) for k in range(C)], 16, quantize_dq_bytes(n), "GB/s",
                        3, proj + " (nf4_quantize_dq)"))
    segs.append(Segment("dequantize", [lambda k=k: q.nf4_dequantize(pk[k], q8[k], c2[k], mu[k], n, torch.bfloat16,
                                                                     out=deq[k]) for k in range(C)],
                        32, dequant_bytes(n), "GB/s", 1, proj + " -> bf16"))
    segs.append(Segment("dequantize_fp32", [lambda k=k: q.nf4_dequantize(pk[k], q8[k], c2[k], mu[k], n,
                                                                          torch.float32, out=deq32[k])
                                            for k in range(C)], 16, dequant_bytes(n, 4), "GB/s", 1,
                        proj + " -> fp32"))
    nodq_b = n // 2 + nb * 4 + n * 2
    segs.append(Segment("dequantize_nodq", [lambda k=k: q.nf4_dequantize(pk[k], None, ab[k], None, n, torch.bfloat16,
                                                                          out=deq[k]) for k in range(C)],
                        32, nodq_b, "GB/s", 1, proj + " -> bf16, fp32 constants (no double quantization)"))

    return wp, dict(pk=pk[0], q8=q8[0], c2=c2[0], mu=mu[0], deq=deq[0], n=n)


def _gemv_segments(q, wl, dev, rank, segs):
    """Config 3: decode GEMV, W 11008 x 4096, r = 16, T in {1, 4, 16}."""
    import torch
    c3 = wl.GEMV_CASES[0]
    W3, _, A3, B3 = wl.linear_inputs(wl.LinearCase(c3.name, 16, c3.K, c3.N, c3.r, c3.scaling,
                                                   rank_seed(c3.seed, rank)))
    st0 = q.quantize_weight(W3.to(dev))
    del W3
    CG = 16  # 16 x 23.7 MB of weights rotate: > 3 x L2
    st3 = [q.QuantState(st0.packed.clone(), st0.absmax_q.clone(), st0.absmax2.clone(), st0.offset.clone(),
                        st0.shape) for _ in range(CG)]
    A3d, B3d = A3.to(dev), B3.to(dev)
    for c in wl.GEMV_CASES:
        g = torch.Generator().manual_seed(rank_seed(c.seed, rank) + c.M)
        xs = [torch.randn(c.M, c.K, generator=g).to(torch.bfloat16).to(dev) for _ in range(CG)]
        ys = [torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev) for _ in range(CG)]
        ws = torch.empty(q.nf4_lora_linear_workspace_size(c.M, c.r), dtype=torch.uint8, device=dev)
        fns = [lambda k=k, xs=xs, ys=ys, ws=ws, c=c: q.nf4_lora_linear_fwd(
            xs[k], st3[k].packed, st3[k].absmax_q, st3[k].absmax2, st3[k].offset, c.N, A3d, B3d, c.scaling,
            y=ys[k], workspace=ws) for k in range(CG)]
        segs.append(Segment(f"gemv_T{c.M}", fns, 32, linear_bytes(c.M, c.K, c.N, c.r), "GB/s", 2,
                            f"x [{c.M},4096] W 11008x4096 NF4+DQ r=16 s=2"))



def _gemm_segment(q, wl, dev, rank, segs, c, tag):
    """Config 4 and the 70B MLP GEMM of config 5."""
    import torch
    cc = wl.LinearCase(c.name, c.M, c.K, c.N, c.r, c.scaling, rank_seed(c.seed, rank))
    W, x, A, B = wl.linear_inputs(cc)
    sts = [q.quantize_weight(W.to(dev)) for _ in range(2)]
    del W
    xs = [x.to(dev), x.to(dev)]
    Ad, Bd = A.to(dev), B.to(dev)
    y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(q.nf4_lora_linear_workspace_size(c.M, c.r), dtype=torch.uint8, device=dev)
    fns = [lambda k=k: q.nf4_lora_linear_fwd(xs[k], sts[k].packed, sts[k].absmax_q, sts[k].absmax2, sts[k].offset,
                                             c.N, Ad, Bd, c.scaling, y=y, workspace=ws) for k in range(2)]
    segs.append(Segment(tag, fns, 2, linear_flops(c.M, c.K, c.N, c.r), "TFLOP/s", 2,
                        f"x [{c.M},{c.K}] W {c.N}x{c.K} NF4+DQ r={c.r} s={c.scaling}"))


def _sweep_segment(q, wl, dev, segs):
    """Config 5: one layer of the 8B-shaped sweep (its 7 weights): quantize +
    double-quantize + dequantize (bf16)."""
    import torch
    Wl = [wl.sweep_weight(0, idx).to(dev).reshape(-1) for idx in range(len(wl.LAYER_8B))]
    bufs = []
    for w in Wl:
        m = w.numel()
        mb = m // BLOCK
        bufs.append((torch.empty(m // 2, dtype=torch.uint8, device=dev),
                     torch.empty(mb, dtype=torch.uint8, device=dev), torch.empty(-(-mb // DQ_BLOCK), device=dev),
                     torch.empty(1, device=dev),
                     torch.empty(q.nf4_quantize_dq_workspace_size(m), dtype=torch.uint8, device=dev),
                     torch.empty(m, dtype=torch.bfloat16, device=dev)))

    def f_layer():
        for w, (p_, q_, c_, o_, wsd, out) in zip(Wl, bufs):
            m = w.numel()
            q.nf4_quantize_dq(w, packed=p_, absmax_q=q_, absmax2=c_, offset=o_, workspace=wsd)
            q.nf4_dequantize(p_, q_, c_, o_, m, torch.bfloat16, out=out)
    layer_b = sum(quantize_dq_bytes(w.numel()) + dequant_bytes(w.numel()) for w in Wl)
    # launches: 3 per quantize + DQ (quantize, run sums, double quantization; 4
    # above 2048 runs: gate, up and down), 1 per dequantize
    layer_launches = sum(4 + (1 if -(-w.numel() // (BLOCK * DQ_BLOCK)) > 2048 else 0) for w in Wl)
    segs.append(Segment("sweep_8B_layer", [f_layer], 1, layer_b, "GB/s", layer_launches,
                        "the 7 linear weights of one 8B-shaped decoder layer (218.1 M params): nf4_quantize_dq + "
                        "nf4_dequantize (bf16); the sweep is 32 such layers"))



def _layer_linear_segments(q, wl, dev, rank, segs):
    """Next row 4: the seven linears of one 8B-shaped decoder layer at M =
    4096 tokens, r = 64, s = 0.25 through the fused NF4 path, and the same
    linears as unquantized bf16 LoRA GEMMs on cuBLAS (torch.matmul; timed for
    the overhead figure only, not counted as this library's launches)."""
    import torch
    M, r, sc = 4096, 64, 0.25
    nf4_fns, bf16_fns, flops = [], [], 0
    for idx, (name, N, K) in enumerate(wl.LAYER_8B):
        W = wl.sweep_weight(0, idx).to(dev)
        g = torch.Generator().manual_seed(rank_seed(wl.sweep_seed(0, idx) + 1, rank))
        x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(dev)
        A = (torch.randn(r, K, generator=g) * 0.01).to(torch.bfloat16).to(dev)
        B = (torch.randn(N, r, generator=g) * 0.01).to(torch.bfloat16).to(dev)
        st = q.quantize_weight(W)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(q.nf4_lora_linear_workspace_size(M, r), dtype=torch.uint8, device=dev)
        nf4_fns.append(lambda x=x, st=st, N=N, A=A, B=B, y=y, ws=ws: q.nf4_lora_linear_fwd(
            x, st.packed, st.absmax_q, st.absmax2, st.offset, N, A, B, sc, y=y, workspace=ws))
        Wt, At, Bt = W.t(), A.t(), B.t()
        yb = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        bf16_fns.append(lambda x=x, Wt=Wt, At=At, Bt=Bt, yb=yb: torch.addmm(torch.matmul(x, Wt), torch.matmul(x, At),
                                                                             Bt, alpha=sc, out=yb))
        flops += linear_flops(M, K, N, r)

    def f_nf4():
        for f in nf4_fns:
            f()

    def f_bf16():
        for f in bf16_fns:
            f()
    cfg = f"the 7 linears of one 8B-shaped decoder layer, M = {M} tokens, r = {r}, s = {sc}"
    segs.append(Segment("layer_8B_linears", [f_nf4], 1, flops, "TFLOP/s", 2 * len(nf4_fns), cfg + ", fused NF4+LoRA"))
    segs.append(Segment("layer_8B_linears_bf16_cublas", [f_bf16], 1, flops, "TFLOP/s", 0,
                        cfg + ", unquantized bf16 LoRA GEMMs on cuBLAS (comparison, not this library)"))


def _bwd_merge_segments(q, wl, dev, rank, segs):
    """Next rows: backward (training shape) and merge + requantize."""
    import torch
    c = wl.GEMM_TRAIN
    W, x, A, B = wl.linear_inputs(wl.LinearCase(c.name, c.M, c.K, c.N, c.r, c.scaling, rank_seed(c.seed, rank)))
    stb = q.quantize_weight(W.to(dev))
    del W
    g = torch.Generator().manual_seed(rank_seed(c.seed, rank) + 7)
    dy = torch.randn(c.M, c.N, generator=g).to(torch.bfloat16).to(dev)
    xd, Ad, Bd = x.to(dev), A.to(dev), B.to(dev)
    dxb = torch.empty(c.M, c.K, dtype=torch.bfloat16, device=dev)
    dAb = torch.empty(c.r, c.K, device=dev)
    dBb = torch.empty(c.N, c.r, device=dev)
    wsb = torch.empty(q.nf4_lora_linear_bwd_workspace_size(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=dev)
    fl_bwd = 2 * c.M * c.N * c.K + 2 * c.M * c.r * (c.N + c.K) + 2 * c.M * c.r * (c.N + c.K) * 2
    segs.append(Segment("backward", [lambda: q.nf4_lora_linear_bwd(
        dy, xd, stb.packed, stb.absmax_q, stb.absmax2, stb.offset, c.K, Ad, Bd, c.scaling, dx=dxb, dA=dAb, dB=dBb,
        workspace=wsb)], 1, fl_bwd, "TFLOP/s", 6,
        f"dx, dA, dB of the training GEMM (g [{c.M},{c.N}], W {c.N}x{c.K}, r={c.r})"))
    m = c.N * c.K
    pko = torch.empty(m // 2, dtype=torch.uint8, device=dev)
    abo = torch.empty(m // BLOCK, device=dev)
    merge_b = dequant_bytes(m, 0) + c.r * c.K * 2 + c.N * c.r * 2 + m // 2 + (m // BLOCK) * 4
    segs.append(Segment("merge", [lambda: q.nf4_merge_requantize(
        stb.packed, stb.absmax_q, stb.absmax2, stb.offset, c.N, c.K, Ad, Bd, c.scaling, packed_out=pko,
        absmax_out=abo)], 1, merge_b, "GB/s", 1, f"merge r={c.r} into W {c.N}x{c.K} and requantize"))


def sharded_segment(q, wl, dev, rank, world):
    """N > 1: quantize + double-quantize one 4096 x 4096 shard per rank of a
    (4096 N) x 4096 tensor, the runs' fp64 sums all-gathered over NCCL so
    that every rank centres on the whole tensor's mean (run eagerly: the
    collective is not captured in a graph)."""
    import torch
    from qlora_nf4_quantize_b200 import sharded
    w = wl.weight((4096, 4096), 0.02, rank_seed(11, rank), "bf16").to(dev).reshape(-1)
    n_total = w.numel() * world

    def f():
        sharded.quantize_sharded(w, n_total, world)
    # launches: quantize, run sums, double quantization (+ chunk sums above 2048 runs); NCCL's are not counted
    launches = 3 + (1 if -(-n_total // (BLOCK * DQ_BLOCK)) > 2048 else 0)
    return Segment("quantize_sharded", [f], 4, quantize_bytes(w.numel()) + dq_bytes(w.numel() // BLOCK), "GB/s",
                   launches, f"one 4096x4096 shard per rank of a {4096 * world}x4096 tensor; run sums all-gathered")


def run_ours(args):
    import torch
    import nf4_workloads as wl
    import qlora_nf4_quantize_b200 as q

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = dist_init(world, "nccl")
    q.lib()  # fails loudly if the CUDA library is missing

    segs, wp, state = build_segments(q, wl, dev, rank, world)
    for s in segs:
        s.capture()
    eager = [sharded_segment(q, wl, dev, rank, world)] if world > 1 else []

    def step(ev=None):
        for j, s in enumerate(segs + eager):
            if ev is not None:
                ev[j][0].record()
            if s.graph is not None:
                s.graph.replay()
            else:
                for r in range(s.reps):
                    s.fns[r % len(s.fns)]()
            if ev is not None:
                ev[j][1].record()

    for _ in range(args.warmup):
        step()
    q.nf4_device_status()
    nseg = len(segs) + len(eager)
    events = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nseg)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record()
    for i in range(args.steps):
        step(events[i])
    t_end.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    q.nf4_device_status()

    K = args.steps
    total_ms = t_start.elapsed_time(t_end)
    seg_ms = [sum(events[i][j][0].elapsed_time(events[i][j][1]) for i in range(K)) for j in range(nseg)]
    red = reduce_max([total_ms] + seg_ms, world, dev)
    total_ms, seg_ms = red[0], red[1:]

    peaks = measured_peaks()

    # -------- end to end through host buffers (rank-local dequant call)
    n = state["n"]
    st_host = [state[k].cpu().pin_memory() for k in ("pk", "q8", "c2", "mu")]
    out_host = torch.empty(n, dtype=torch.bfloat16).pin_memory()
    dev_in = [torch.empty_like(t, device=dev) for t in st_host]
    e2e_iters = max(10, min(K, 100))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for it in range(e2e_iters + 3):
        if it == 3:
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize()
            e0.record()
        for d, h in zip(dev_in, st_host):
            d.copy_(h, non_blocking=True)
        q.nf4_dequantize(dev_in[0], dev_in[1], dev_in[2], dev_in[3], n, torch.bfloat16, out=state["deq"])
        out_host.copy_(state["deq"], non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = reduce_max([e0.elapsed_time(e1) / e2e_iters], world, dev)[0]
    h2d = sum(t.numel() * t.element_size() for t in st_host)
    d2h = out_host.numel() * 2

    # the timed region lasts well under a second: every kernel runs at the
    # burst clocks, so fractions are of the burst peaks
    tflops_peak = peaks["bf16_tflops"] if total_ms < 1000 else peaks["bf16_tflops_sustained"]
    kernels = []
    by = {}
    for s, ms in zip(segs + eager, seg_ms):
        us = ms / (K * s.reps) * 1e3
        if s.unit == "GB/s":
            ach, peak = s.work / (us * 1e-6) / 1e9, peaks["hbm_gbs"]
        else:
            ach, peak = s.work / (us * 1e-6) / 1e12, tflops_peak
        e = {"call": s.name, "us": round(us, 3), "achieved": round(ach, 2), "unit": s.unit, "peak": peak,
             "frac": round(ach / peak, 4), "work_per_call": s.work, "calls_per_step": s.reps,
             "config": s.config}
        if s.name == "sweep_8B_layer":
            e["sweep_32_layers_s"] = round(us * wl.N_LAYERS_8B * 1e-6, 5)
        kernels.append(e)
        by[s.name] = e
    if "layer_8B_linears" in by and "layer_8B_linears_bf16_cublas" in by:
        by["layer_8B_linears"]["overhead_vs_bf16_lora"] = round(
            by["layer_8B_linears"]["us"] / by["layer_8B_linears_bf16_cublas"]["us"] - 1, 4)
    launches = sum(s.reps * s.launches for s in segs + eager) * K

    if rank != 0:
        return
    deq = by["dequantize"]
    gemm = by["gemm_M4096"]
    line = {
        "metric": METRIC, "value": round(world * deq["achieved"], 2), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(total_ms / K, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(world),
        "roofline": {"bound": "tensor", "kernel": "k_gemm_tc (nf4_lora_linear_fwd, M=4096: training GEMM)",
                     "achieved": gemm["achieved"], "peak": tflops_peak, "unit": "TFLOP/s",
                     "frac": round(gemm["achieved"] / tflops_peak, 4),
                     "traffic": recorded_traffic("gemm_tc.cu"),
                     "peak_source": peaks["source"] + (" bf16 burst (timed region < 1 s)" if total_ms < 1000
                                                       else " bf16 sustained (timed region >= 1 s)")},
        "kernels": kernels,
        "e2e": {"value": round(world * dequant_bytes(n) / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": "nf4_dequantize with pinned host inputs and output"},
        "gpu_launches": launches,
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wp)
    print(json.dumps(line), flush=True)


def bench_config(world):
    return {"workload": WORKLOAD, "quant": "NF4 block 64 + double quant block 256 (E4M3, centred)",
            "arith": "quantize/dequantize fp32 -> bf16; linear bf16 x bf16 tensor cores, fp32 accumulate",
            "timing": "each call replayed back to back from a CUDA graph, events around each call's replays",
            "l2": "inputs rotate over copies larger than the 126 MB L2 (no call reads a warm input)",
            "parallelism": f"independent replicas x{world} + one sharded tensor" if world > 1 else "single GPU"}


# ------------------------------------------------------------------ CPU oracle
def oracle_dequant_rate(wp, budget_s):
    """The oracle's NF4 dequant (bf16 output) on the projection weight,
    repeated for about budget_s seconds; returns (GB/s, repetitions)."""
    import torch
    import oracle
    bits = wp.contiguous().view(torch.int16).numpy().view(np.uint16).ravel()
    packed, c1 = oracle.quantize(bits)
    codes, c2, mu = oracle.double_quantize(c1)
    n = bits.size
    oracle.dequantize(packed, codes, c2, mu, n, "bf16")  # first call: one-time setup, untimed
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.dequantize(packed, codes, c2, mu, n, "bf16")
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return reps * dequant_bytes(n) / el / 1e9, reps, el


def _oracle_slice_worker(job):
    """One host process: the oracle's dequant of one slice of the quantized
    state (whole runs of 256 blocks), repeated for budget_s seconds."""
    packed, codes, c2, mu, n, budget_s = job
    import oracle
    oracle.dequantize(packed, codes, c2, mu, n, "bf16")  # first call: one-time setup, untimed
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.dequantize(packed, codes, c2, mu, n, "bf16")
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return reps, n, el


def oracle_dequant_rate_cores(wp, budget_s, cores):
    """The oracle's dequant on `cores` host processes at once (spawned, each a
    slice of the weight on run boundaries); returns (GB/s, bytes moved)."""
    import multiprocessing as mp
    import torch
    import oracle
    bits = wp.contiguous().view(torch.int16).numpy().view(np.uint16).ravel()
    packed, c1 = oracle.quantize(bits)
    codes, c2, mu = oracle.double_quantize(c1)
    n = bits.size
    run = BLOCK * DQ_BLOCK
    runs = -(-n // run)
    jobs = []
    for i in range(cores):
        r0, r1 = runs * i // cores, runs * (i + 1) // cores
        e0, e1 = r0 * run, min(r1 * run, n)
        if e1 <= e0:
            continue
        jobs.append((packed[e0 // 2:(e1 + 1) // 2].copy(), codes[e0 // BLOCK:-(-e1 // BLOCK)].copy(),
                     c2[r0:r1].copy(), mu, e1 - e0, budget_s))
    ctx = mp.get_context("spawn")
    with ctx.Pool(len(jobs)) as pool:
        res = pool.map(_oracle_slice_worker, jobs)
    # the processes run side by side for the same budget: rates add up
    return sum(reps * dequant_bytes(m) / el for reps, m, el in res) / 1e9, len(jobs)


def host_cores():
    """Host cores the oracle may use (the host is shared: at most 16)."""
    return max(1, min(16, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)))


def cpu_baseline(wp, budget_s=10.0):
    gbs1, reps, el = oracle_dequant_rate(wp, budget_s * 0.4)
    cores = host_cores()
    gbs, used = oracle_dequant_rate_cores(wp, budget_s * 0.6, cores) if cores > 1 else (gbs1, 1)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": used, "kind": "oracle", "value_1core": round(gbs1, 4),
            "sample": f"oracle nf4 dequantize (bf16 out) of the 4096x4096 projection weight: {used} host processes "
                      f"on slices of whole 256-block runs for {budget_s * 0.6:.0f} s; single thread {reps} full "
                      f"passes in {el:.1f} s (value_1core)"}


def run_reference(args):
    """The reference arm: the CPU oracle (the method's plain C restatement),
    as it stands, on the host cores of rank 0 (other ranks exit at once).
    Each step is one single-threaded oracle dequantize of the whole
    projection weight to bf16 (the call the metric's headline value times);
    the oracle quantizes the weight once, outside the timed region."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch
    import nf4_workloads as wl
    import oracle
    wp = wl.weight((4096, 4096), 0.02, wl.PROJECTION["seed"], "bf16", outliers=True)
    bits = wp.contiguous().view(torch.int16).numpy().view(np.uint16).ravel()
    packed, c1 = oracle.quantize(bits)
    codes, c2, mu = oracle.double_quantize(c1)
    n = bits.size
    for _ in range(max(1, args.warmup)):
        oracle.dequantize(packed, codes, c2, mu, n, "bf16")
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.dequantize(packed, codes, c2, mu, n, "bf16")
    el = time.perf_counter() - t0
    value = args.steps * dequant_bytes(n) / el / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": bench_config(world),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{args.steps} full dequantize passes (bf16 out) of the 4096x4096 projection "
                                       f"weight, single thread (state quantized once by the oracle, outside the "
                                       f"timed region); the oracle has no GPU kernels, so only the headline call "
                                       f"of the workload is timed"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ isolated per-call suite
def graph_us(fn, reps, warm=3, trials=3):
    """Median over `trials` of the per-call time (us) of `reps` calls of
    `fn` captured in one CUDA graph and replayed (no launch gaps)."""
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(trials):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        g.replay()
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e) * 1e3 / reps)
    del g
    return sorted(times)[len(times) // 2]


def run_suite(args):
    """Every call of the path timed in isolation (CUDA graphs, inputs rotating
    over copies larger than L2), with and without double quantization, plus
    the 8B-shaped whole-model sweep and one decoder layer's linears through
    the fused NF4 path against unquantized bf16 LoRA GEMMs (torch.matmul on
    cuBLAS).  One JSON line per measurement on rank 0."""
    import torch
    import nf4_workloads as wl
    import qlora_nf4_quantize_b200 as q

    rank, world, local = dist_env()
    if rank != 0:
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    q.lib()
    peaks = measured_peaks()

    def emit(name, us, work, unit, **extra):
        if unit == "GB/s":
            ach, peak = work / (us * 1e-6) / 1e9, peaks["hbm_gbs"]
        else:
            ach, peak = work / (us * 1e-6) / 1e12, peaks["bf16_tflops"]
        line = {"suite": name, "us": round(us, 3), "achieved": round(ach, 2), "unit": unit, "peak": peak,
                "frac": round(ach / peak, 4), "work_per_call": work, "timing": "CUDA graph, isolated call"}
        line.update(extra)
        print(json.dumps(line), flush=True)

    sections = set(args.sections.split(",")) if args.sections else None

    def want(name):
        return sections is None or name in sections

    rot = [0]

    def nxt(c):
        rot[0] += 1
        return rot[0] % c

    if want("projection"):
        # ---- projection 4096x4096 bf16: quantize, double-quantize, dequantize (with / without DQ)
        wp = wl.weight_case(wl.PROJECTION).to(dev).reshape(-1)
        n, C = wp.numel(), 6
        nb = n // BLOCK
        Ws = [wp.clone() for _ in range(C)]
        sts = [q.quantize_weight(w) for w in Ws]
        raw = [q.nf4_quantize(w) for w in Ws[:C]]  # (packed, fp32 absmax): the no-DQ state
        absb = [torch.empty(nb, device=dev) for _ in range(C)]
        outs = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(C)]
        outs32 = [torch.empty(n, dtype=torch.float32, device=dev) for _ in range(C)]
        q8s = [torch.empty(nb, dtype=torch.uint8, device=dev) for _ in range(C)]
        c2s = [torch.empty(-(-nb // DQ_BLOCK), device=dev) for _ in range(C)]
        offs = [torch.empty(1, device=dev) for _ in range(C)]
        ws = torch.empty(q.nf4_double_quantize_workspace_size(nb), dtype=torch.uint8, device=dev)

        def f_quant():
            k = nxt(C)
            q.nf4_quantize(Ws[k], packed=sts[k].packed, absmax=absb[k])

        def f_dq():
            k = nxt(C)
            q.nf4_double_quantize(absb[k], absmax_q=q8s[k], absmax2=c2s[k], offset=offs[k], workspace=ws)

        def f_deq(dq, f32):
            def f():
                k = nxt(C)
                o = outs32[k] if f32 else outs[k]
                if dq:
                    st = sts[k]
                    q.nf4_dequantize(st.packed, st.absmax_q, st.absmax2, st.offset, n,
                                     torch.float32 if f32 else torch.bfloat16, out=o)
                else:
                    q.nf4_dequantize(raw[k][0], None, raw[k][1], None, n, torch.float32 if f32 else torch.bfloat16,
                                     out=o)
            return f

        proj = "projection 4096x4096 bf16"
        emit(f"quantize {proj}", graph_us(f_quant, 20), quantize_bytes(n), "GB/s")
        emit(f"double_quantize {nb} constants", graph_us(f_dq, 20), dq_bytes(nb), "GB/s")
        emit(f"dequantize {proj} -> bf16, DQ", graph_us(f_deq(True, False), 20), dequant_bytes(n), "GB/s")
        emit(f"dequantize {proj} -> fp32, DQ", graph_us(f_deq(True, True), 20), dequant_bytes(n, 4), "GB/s")
        nodq_b = n // 2 + nb * 4 + n * 2
        emit(f"dequantize {proj} -> bf16, no DQ (fp32 c1)", graph_us(f_deq(False, False), 20), nodq_b, "GB/s",
             bytes_per_param=round(nodq_b / n - 2, 6))
        del Ws, sts, raw, absb, outs, outs32, q8s, c2s, offs
        torch.cuda.empty_cache()

    if want("linear"):
        # ---- fused linear: decode GEMV and tensor-core GEMM, with / without DQ
        def linear_case(c, dq, copies, reps):
            W, x, A, B = wl.linear_inputs(c)
            Wd = W.to(dev)
            stl = [q.quantize_weight(Wd, double_quant=dq) for _ in range(copies)]
            del W, Wd
            xd, Ad, Bd = x.to(dev), A.to(dev), B.to(dev)
            y = torch.empty(c.M, c.N, dtype=torch.bfloat16, device=dev)
            wsl = torch.empty(max(1, q.nf4_lora_linear_workspace_size(c.M, c.r)), dtype=torch.uint8, device=dev)

            def f():
                st = stl[nxt(copies)]
                q.nf4_lora_linear_fwd(xd, st.packed, st.absmax_q, st.absmax2, st.offset, c.N, Ad, Bd, c.scaling,
                                      y=y, workspace=wsl)
            us = graph_us(f, reps)
            q.nf4_device_status()
            wb = c.N * c.K // 2 + (c.N * c.K // BLOCK) * (1 if dq else 4) + (-(-(c.N * c.K // BLOCK) // DQ_BLOCK) * 4 + 4
                                                                              if dq else 0)
            byts = wb + c.M * c.K * 2 + c.r * c.K * 2 + c.N * c.r * 2 + c.M * c.N * 2
            return us, byts

        for c in wl.GEMV_CASES:
            for dq in (True, False):
                us, byts = linear_case(c, dq, 8, 20)
                emit(f"{c.name}{'' if dq else ', no DQ'}", us, byts, "GB/s",
                     tflops=round(linear_flops(c.M, c.K, c.N, c.r) / (us * 1e-6) / 1e12, 3))
        for c in (wl.GEMM_TRAIN, wl.GEMM_70B_MLP):
            for dq in (True, False):
                us, _ = linear_case(c, dq, 1, 5)
                emit(f"{c.name}{'' if dq else ', no DQ'}", us, linear_flops(c.M, c.K, c.N, c.r), "TFLOP/s",
                     peak_sustained=peaks["bf16_tflops_sustained"])
        torch.cuda.empty_cache()

    if want("backward"):
        # ---- backward through the frozen base: dx (fused NF4 GEMM) and the adapter gradients
        for c in (wl.GEMM_TRAIN, wl.GEMM_70B_MLP):
            W, x, A, B = wl.linear_inputs(c)
            g = torch.Generator().manual_seed(c.seed + 7)
            dy = torch.randn(c.M, c.N, generator=g).to(torch.bfloat16).to(dev)
            st = q.quantize_weight(W.to(dev))
            xd, Ad, Bd = x.to(dev), A.to(dev), B.to(dev)
            dxb = torch.empty(c.M, c.K, dtype=torch.bfloat16, device=dev)
            dAb = torch.empty(c.r, c.K, device=dev)
            dBb = torch.empty(c.N, c.r, device=dev)
            wsb = torch.empty(q.nf4_lora_linear_bwd_workspace_size(c.M, c.N, c.K, c.r), dtype=torch.uint8, device=dev)

            def f_dx():
                q.nf4_lora_linear_bwd(dy, None, st.packed, st.absmax_q, st.absmax2, st.offset, c.K, Ad, Bd, c.scaling,
                                      want=("dx",), dx=dxb, workspace=wsb)

            def f_grads():
                q.nf4_lora_linear_bwd(dy, xd, st.packed, st.absmax_q, st.absmax2, st.offset, c.K, Ad, Bd, c.scaling,
                                      want=("dA", "dB"), dA=dAb, dB=dBb, workspace=wsb)

            def f_all():
                q.nf4_lora_linear_bwd(dy, xd, st.packed, st.absmax_q, st.absmax2, st.offset, c.K, Ad, Bd, c.scaling,
                                      dx=dxb, dA=dAb, dB=dBb, workspace=wsb)
            us_dx, us_gr, us_all = graph_us(f_dx, 3), graph_us(f_grads, 3), graph_us(f_all, 3)
            q.nf4_device_status()
            fl_dx = 2 * c.M * c.N * c.K + 2 * c.M * c.r * (c.N + c.K)
            fl_gr = 2 * c.M * c.r * (c.N + c.K) * 2  # two down-projections + the two gradient products
            emit(f"backward dx {c.name}", us_dx, fl_dx, "TFLOP/s", peak_sustained=peaks["bf16_tflops_sustained"])
            emit(f"backward dA + dB {c.name}", us_gr, fl_gr, "TFLOP/s")
            emit(f"backward dx + dA + dB {c.name}", us_all, fl_dx + fl_gr, "TFLOP/s")
            del W, x, A, B, dy, st, xd, Ad, Bd, dxb, dAb, dBb, wsb
            torch.cuda.empty_cache()

    if want("merge"):
        # ---- merge the adapter into the quantized base and requantize (+ double
        # quantization of the new constants), and the error the requantization adds
        for c in (wl.GEMM_TRAIN, wl.GEMM_70B_MLP):
            W, _, A, B = wl.linear_inputs(c)
            Wd, Ad, Bd = W.to(dev), A.to(dev), B.to(dev)
            st = q.quantize_weight(Wd)
            m = c.N * c.K
            pk = torch.empty(m // 2, dtype=torch.uint8, device=dev)
            ab = torch.empty(m // BLOCK, device=dev)

            def f_merge():
                q.nf4_merge_requantize(st.packed, st.absmax_q, st.absmax2, st.offset, c.N, c.K, Ad, Bd, c.scaling,
                                       packed_out=pk, absmax_out=ab)
            us = graph_us(f_merge, 3)
            byts = dequant_bytes(m, 0) + c.r * c.K * 2 + c.N * c.r * 2 + m // 2 + (m // BLOCK) * 4
            merged = q.merge_and_requantize(st, Ad, Bd, c.scaling)
            w_base = q.nf4_dequantize(st.packed, st.absmax_q, st.absmax2, st.offset, m, torch.float32).view(c.N, c.K)
            w_new = q.nf4_dequantize(merged.packed, merged.absmax_q, merged.absmax2, merged.offset, m,
                                     torch.float32).view(c.N, c.K)
            delta = c.scaling * (Bd.float() @ Ad.float())
            w_exact = w_base + delta
            rms = lambda t: float(t.pow(2).mean().sqrt())
            emit(f"merge + requantize {c.N}x{c.K} r={c.r}", us, byts, "GB/s",
                 fma_per_s=round(m * c.r / (us * 1e-6) / 1e12, 3), fma_unit="T fma/s (fp32 chain)",
                 base_quant_rel_rms=round(rms(w_base - Wd.float()) / rms(Wd.float()), 6),
                 requant_rel_rms=round(rms(w_new - w_exact) / rms(w_exact), 6),
                 adapter_rel_rms=round(rms(delta) / rms(w_base), 6),
                 adapter_retained=round(float(((w_new - w_base) * delta).sum() / (delta * delta).sum()), 4))
            del W, Wd, Ad, Bd, st, pk, ab, merged, w_base, w_new, delta, w_exact
            torch.cuda.empty_cache()

    if want("layer"):
        # ---- one 8B-shaped decoder layer, M = 4096 tokens, r = 64, s = 0.25:
        # fused NF4 + LoRA against bf16 x W^T + s (x A^T) B^T on cuBLAS
        M, r, sc = 4096, 64, 0.25
        t_nf4 = t_bf16 = 0.0
        flops = 0
        for idx, (name, N, K) in enumerate(wl.LAYER_8B):
            W = wl.sweep_weight(0, idx).to(dev)
            g = torch.Generator().manual_seed(wl.sweep_seed(0, idx) + 1)
            x = torch.randn(M, K, generator=g).to(torch.bfloat16).to(dev)
            A = (torch.randn(r, K, generator=g) * 0.01).to(torch.bfloat16).to(dev)
            B = (torch.randn(N, r, generator=g) * 0.01).to(torch.bfloat16).to(dev)
            st = q.quantize_weight(W)
            y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            wsl = torch.empty(q.nf4_lora_linear_workspace_size(M, r), dtype=torch.uint8, device=dev)
            Wt, At, Bt = W.t(), A.t(), B.t()

            def f_nf4():
                q.nf4_lora_linear_fwd(x, st.packed, st.absmax_q, st.absmax2, st.offset, N, A, B, sc, y=y, workspace=wsl)

            def f_bf16():
                yb = torch.matmul(x, Wt)
                torch.addmm(yb, torch.matmul(x, At), Bt, alpha=sc, out=y)

            a_us, b_us = graph_us(f_nf4, 3), graph_us(f_bf16, 3)
            fl = linear_flops(M, K, N, r)
            emit(f"layer {name} {N}x{K} M={M} r={r}: fused NF4+LoRA", a_us, fl, "TFLOP/s",
                 bf16_lora_us=round(b_us, 3), ratio_nf4_over_bf16=round(a_us / b_us, 4))
            t_nf4, t_bf16, flops = t_nf4 + a_us, t_bf16 + b_us, flops + fl
            del W, x, A, B, st, y, wsl
        emit(f"8B decoder layer (7 linears) M={M} r={r}: fused NF4+LoRA", t_nf4, flops, "TFLOP/s",
             bf16_lora_us=round(t_bf16, 3), overhead_vs_bf16=round(t_nf4 / t_bf16 - 1, 4),
             note="forward linears only; the pages' 25-40 % slowdown figure is per training step")
        torch.cuda.empty_cache()

    if want("sweep"):
        # ---- 8B-shaped whole-model sweep: quantize + DQ + dequantize of every
        # linear weight, layer by layer (layer 0's seeded weights stand in for all
        # 32 layers: the same shapes and work; 224 weights, 6.98e9 parameters)
        Wl = [wl.sweep_weight(0, idx).to(dev).reshape(-1) for idx in range(len(wl.LAYER_8B))]
        bufs = []
        for w in Wl:
            m = w.numel()
            mb = m // BLOCK
            bufs.append((torch.empty(m // 2, dtype=torch.uint8, device=dev), torch.empty(mb, device=dev),
                         torch.empty(mb, dtype=torch.uint8, device=dev), torch.empty(-(-mb // DQ_BLOCK), device=dev),
                         torch.empty(1, device=dev),
                         torch.empty(q.nf4_double_quantize_workspace_size(mb), dtype=torch.uint8, device=dev),
                         torch.empty(m, dtype=torch.bfloat16, device=dev)))

        def f_layer():
            for w, (pk, ab, q8, c2, off, wsd, out) in zip(Wl, bufs):
                m = w.numel()
                q.nf4_quantize(w, packed=pk, absmax=ab)
                q.nf4_double_quantize(ab, absmax_q=q8, absmax2=c2, offset=off, workspace=wsd)
                q.nf4_dequantize(pk, q8, c2, off, m, torch.bfloat16, out=out)

        layer_us = graph_us(f_layer, 4)
        per_layer = sum(quantize_bytes(w.numel()) + dq_bytes(w.numel() // BLOCK) + dequant_bytes(w.numel()) for w in Wl)
        L = wl.N_LAYERS_8B
        emit(f"8B-shaped sweep: quantize + DQ + dequantize, {L} layers x 7 linears", layer_us * L, per_layer * L,
             "GB/s", params=sum(w.numel() for w in Wl) * L, seconds=round(layer_us * L * 1e-6, 4))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1600)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sections", default="",
                    help="with --suite: comma-separated subset of projection,linear,backward,merge,layer,sweep")
    ap.add_argument("--suite", action="store_true",
                    help="time every call in isolation (no-DQ variant, sweep, decoder layer); one line each")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
        return
    if args.suite:
        run_suite(args)
        return
    run_ours(args)
    rank, world, _ = dist_env()
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
