"""ctypes binding of libnf4.so: argument marshalling only.

Each function takes torch tensors, checks their device/dtype/shape, allocates
outputs that were not supplied (torch owns all device memory), and calls the
C entry point of the same name on the current CUDA stream.  Nothing here
computes: a call either reaches the CUDA library or raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# NF4_LIB_PATH selects another build of the same library (alternative kernel
# configurations built with build.build(out=..., defines=...)).
LIB_PATH = os.environ.get("NF4_LIB_PATH", os.path.join(_PKG, "libnf4.so"))
BLOCKSIZE = 64
DQ_BLOCKSIZE = 256

_STATUS = {0: "NF4_OK", 1: "NF4_ERR_INVALID", 2: "NF4_ERR_UNSUPPORTED", 3: "NF4_ERR_CUDA", 4: "NF4_ERR_TIMEOUT"}
_F32, _BF16 = 0, 1
_lib = None


class Nf4Error(RuntimeError):
    def __init__(self, fn: str, status: int, cuda_error: int = 0):
        self.status = status
        msg = f"{fn} returned {_STATUS.get(status, status)}"
        if status == 3:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


def lib() -> ctypes.CDLL:
    """Load libnf4.so from the package directory (raises if it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} not built; run python -m qlora_nf4_quantize_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    P, i64, i32, f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
    L.nf4_status_string.restype = ctypes.c_char_p
    L.nf4_status_string.argtypes = [i32]
    L.nf4_last_cuda_error.restype = i32
    L.nf4_codebook.restype = i32
    L.nf4_codebook.argtypes = [P]
    L.nf4_quantize.restype = i32
    L.nf4_quantize.argtypes = [P, i32, i64, i32, P, P, P]
    L.nf4_double_quantize_workspace_size.restype = i64
    L.nf4_double_quantize_workspace_size.argtypes = [i64, i32]
    L.nf4_double_quantize.restype = i32
    L.nf4_double_quantize.argtypes = [P, i64, i32, P, P, P, P, i64, P]
    L.nf4_quantize_dq_workspace_size.restype = i64
    L.nf4_quantize_dq_workspace_size.argtypes = [i64, i32, i32]
    L.nf4_quantize_dq.restype = i32
    L.nf4_quantize_dq.argtypes = [P, i32, i64, i32, i32, P, P, P, P, P, i64, P]
    L.nf4_dq_run_sums.restype = i32
    L.nf4_dq_run_sums.argtypes = [P, i64, i32, P, P]
    L.nf4_double_quantize_sharded_workspace_size.restype = i64
    L.nf4_double_quantize_sharded_workspace_size.argtypes = [i64, i32]
    L.nf4_double_quantize_sharded.restype = i32
    L.nf4_double_quantize_sharded.argtypes = [P, i64, i32, P, i64, P, P, P, P, i64, P]
    L.nf4_dequantize.restype = i32
    L.nf4_dequantize.argtypes = [P, P, P, P, i64, i32, i32, P, i32, P]
    L.nf4_lora_linear_workspace_size.restype = i64
    L.nf4_lora_linear_workspace_size.argtypes = [i64, i32]
    L.nf4_lora_linear_fwd.restype = i32
    L.nf4_lora_linear_fwd.argtypes = [P, i64, i64, i64, P, P, P, P, P, P, i32, f32, P, P, i64, P]
    L.nf4_lora_linear_fwd_noalloc.restype = i32
    L.nf4_lora_linear_fwd_noalloc.argtypes = [P, i64, i64, i64, P, P, P, P, P, P, i32, f32, P, P]
    L.nf4_device_status.restype = i32
    L.nf4_device_status.argtypes = [P]
    L.nf4_lora_linear_bwd_workspace_size.restype = i64
    L.nf4_lora_linear_bwd_workspace_size.argtypes = [i64, i64, i64, i32]
    L.nf4_lora_linear_bwd.restype = i32
    L.nf4_lora_linear_bwd.argtypes = [P, P, i64, i64, i64, P, P, P, P, P, P, i32, f32, P, P, P, P, i64, P]
    L.nf4_merge_requantize.restype = i32
    L.nf4_merge_requantize.argtypes = [P, P, P, P, i64, i64, P, P, i32, f32, P, P, P]
    L.nf4_selftest_wait_timeout.restype = i32
    L.nf4_selftest_wait_timeout.argtypes = [i64, P]
    _lib = L
    return L


def _check(fn: str, status: int):
    if status != 0:
        raise Nf4Error(fn, status, lib().nf4_last_cuda_error())


def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None, numel=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if numel is not None and t.numel() != numel:
        raise ValueError(f"{name} must have {numel} elements, got {t.numel()}")


def nf4_codebook() -> torch.Tensor:
    out = torch.empty(16, dtype=torch.float32)
    _check("nf4_codebook", lib().nf4_codebook(_p(out)))
    return out


def nf4_quantize(w: torch.Tensor, blocksize: int = BLOCKSIZE, packed=None, absmax=None, stream=None):
    """Blockwise NF4 quantization of a flattened fp32/bf16 CUDA tensor.
    Returns (packed uint8[n/2], absmax fp32[ceil(n/64)])."""
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("w must be float32 or bfloat16")
    _need(w, "w")
    n = w.numel()
    nb = (n + blocksize - 1) // blocksize
    packed = torch.empty(n // 2, dtype=torch.uint8, device=w.device) if packed is None else packed
    absmax = torch.empty(nb, dtype=torch.float32, device=w.device) if absmax is None else absmax
    _need(packed, "packed", torch.uint8, n // 2)
    _need(absmax, "absmax", torch.float32, nb)
    st = lib().nf4_quantize(_p(w), _BF16 if w.dtype == torch.bfloat16 else _F32, n, blocksize, _p(packed),
                            _p(absmax), _stream(stream))
    _check("nf4_quantize", st)
    return packed, absmax


def nf4_double_quantize_workspace_size(nblocks: int, dq_blocksize: int = DQ_BLOCKSIZE) -> int:
    return int(lib().nf4_double_quantize_workspace_size(nblocks, dq_blocksize))


def nf4_double_quantize(absmax: torch.Tensor, dq_blocksize: int = DQ_BLOCKSIZE, centre: bool = True,
                        absmax_q=None, absmax2=None, offset=None, workspace=None, stream=None):
    """Returns (absmax_q uint8[nb], absmax2 fp32[ceil(nb/256)], offset fp32[1] or None)."""
    _need(absmax, "absmax", torch.float32)
    nb = absmax.numel()
    nd = (nb + dq_blocksize - 1) // dq_blocksize
    dev = absmax.device
    absmax_q = torch.empty(nb, dtype=torch.uint8, device=dev) if absmax_q is None else absmax_q
    absmax2 = torch.empty(nd, dtype=torch.float32, device=dev) if absmax2 is None else absmax2
    if centre and offset is None:
        offset = torch.empty(1, dtype=torch.float32, device=dev)
    if not centre:
        offset = None
    ws_bytes = nf4_double_quantize_workspace_size(nb, dq_blocksize) if centre else 0
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = lib().nf4_double_quantize(_p(absmax), nb, dq_blocksize, _p(absmax_q), _p(absmax2), _p(offset),
                                   _p(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check("nf4_double_quantize", st)
    return absmax_q, absmax2, offset


def nf4_quantize_dq_workspace_size(n: int, blocksize: int = BLOCKSIZE, dq_blocksize: int = DQ_BLOCKSIZE) -> int:
    return int(lib().nf4_quantize_dq_workspace_size(n, blocksize, dq_blocksize))


def nf4_quantize_dq(w: torch.Tensor, centre: bool = True, packed=None, absmax_q=None, absmax2=None, offset=None,
                    workspace=None, stream=None):
    """NF4 quantization and double quantization in one call.  Returns
    (packed uint8[n/2], absmax_q uint8[nb], absmax2 fp32[ceil(nb/256)],
    offset fp32[1] or None)."""
    if w.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("w must be float32 or bfloat16")
    _need(w, "w")
    n = w.numel()
    nb = (n + BLOCKSIZE - 1) // BLOCKSIZE
    nd = (nb + DQ_BLOCKSIZE - 1) // DQ_BLOCKSIZE
    dev = w.device
    packed = torch.empty(n // 2, dtype=torch.uint8, device=dev) if packed is None else packed
    absmax_q = torch.empty(nb, dtype=torch.uint8, device=dev) if absmax_q is None else absmax_q
    absmax2 = torch.empty(nd, dtype=torch.float32, device=dev) if absmax2 is None else absmax2
    if centre and offset is None:
        offset = torch.empty(1, dtype=torch.float32, device=dev)
    if not centre:
        offset = None
    _need(packed, "packed", torch.uint8, n // 2)
    _need(absmax_q, "absmax_q", torch.uint8, nb)
    _need(absmax2, "absmax2", torch.float32, nd)
    if workspace is None:
        workspace = torch.empty(max(16, nf4_quantize_dq_workspace_size(n)), dtype=torch.uint8, device=dev)
    st = lib().nf4_quantize_dq(_p(w), _BF16 if w.dtype == torch.bfloat16 else _F32, n, BLOCKSIZE, DQ_BLOCKSIZE,
                               _p(packed), _p(absmax_q), _p(absmax2), _p(offset), _p(workspace),
                               workspace.numel() * workspace.element_size(), _stream(stream))
    _check("nf4_quantize_dq", st)
    return packed, absmax_q, absmax2, offset


def nf4_dq_run_sums(absmax: torch.Tensor, dq_blocksize: int = DQ_BLOCKSIZE, out=None, stream=None) -> torch.Tensor:
    """fp64 sum of each run of 256 constants (the first step of the centring
    mean); returns float64[ceil(nb / 256)]."""
    _need(absmax, "absmax", torch.float32)
    nb = absmax.numel()
    nd = (nb + dq_blocksize - 1) // dq_blocksize
    out = torch.empty(nd, dtype=torch.float64, device=absmax.device) if out is None else out
    _need(out, "out", torch.float64, nd)
    _check("nf4_dq_run_sums", lib().nf4_dq_run_sums(_p(absmax), nb, dq_blocksize, _p(out), _stream(stream)))
    return out


def nf4_double_quantize_sharded(absmax: torch.Tensor, run_sums_all: torch.Tensor, nblocks_total: int,
                                dq_blocksize: int = DQ_BLOCKSIZE, absmax_q=None, absmax2=None, offset=None,
                                workspace=None, stream=None):
    """Double quantization of one shard with the mean of the whole tensor
    (run_sums_all: every run's fp64 sum, in shard order).  Returns
    (absmax_q uint8[nb], absmax2 fp32[ceil(nb/256)], offset fp32[1])."""
    _need(absmax, "absmax", torch.float32)
    nb = absmax.numel()
    nd = (nb + dq_blocksize - 1) // dq_blocksize
    nd_total = (nblocks_total + dq_blocksize - 1) // dq_blocksize
    _need(run_sums_all, "run_sums_all", torch.float64, nd_total)
    dev = absmax.device
    absmax_q = torch.empty(nb, dtype=torch.uint8, device=dev) if absmax_q is None else absmax_q
    absmax2 = torch.empty(nd, dtype=torch.float32, device=dev) if absmax2 is None else absmax2
    offset = torch.empty(1, dtype=torch.float32, device=dev) if offset is None else offset
    ws_bytes = int(lib().nf4_double_quantize_sharded_workspace_size(nblocks_total, dq_blocksize))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    st = lib().nf4_double_quantize_sharded(_p(absmax), nb, dq_blocksize, _p(run_sums_all), nblocks_total,
                                           _p(absmax_q), _p(absmax2), _p(offset), _p(workspace),
                                           workspace.numel() * workspace.element_size(), _stream(stream))
    _check("nf4_double_quantize_sharded", st)
    return absmax_q, absmax2, offset


def nf4_dequantize(packed: torch.Tensor, absmax_q: Optional[torch.Tensor], absmax2: torch.Tensor,
                   offset: Optional[torch.Tensor], n: int, out_dtype=torch.bfloat16, blocksize: int = BLOCKSIZE,
                   dq_blocksize: int = DQ_BLOCKSIZE, out=None, stream=None) -> torch.Tensor:
    """Dequantize to a flat fp32/bf16 tensor of n elements.  absmax_q None:
    absmax2 holds the fp32 first-level constants (no double quantization)."""
    _need(packed, "packed", torch.uint8, n // 2)
    _need(absmax2, "absmax2", torch.float32)
    if absmax_q is not None:
        _need(absmax_q, "absmax_q", torch.uint8)
    if out is None:
        out = torch.empty(n, dtype=out_dtype, device=packed.device)
    _need(out, "out", out_dtype, n)
    st = lib().nf4_dequantize(_p(packed), _p(absmax_q), _p(absmax2), _p(offset), n, blocksize, dq_blocksize,
                              _p(out), _BF16 if out_dtype == torch.bfloat16 else _F32, _stream(stream))
    _check("nf4_dequantize", st)
    return out


def nf4_lora_linear_workspace_size(M: int, r: int) -> int:
    return int(lib().nf4_lora_linear_workspace_size(M, r))


def nf4_lora_linear_fwd(x: torch.Tensor, packed: torch.Tensor, absmax_q: Optional[torch.Tensor],
                        absmax2: torch.Tensor, offset: Optional[torch.Tensor], N: int,
                        A: Optional[torch.Tensor] = None, B: Optional[torch.Tensor] = None, scaling: float = 1.0,
                        y=None, workspace=None, stream=None) -> torch.Tensor:
    """y[M, N] = x W~^T + scaling (x A^T) B^T with W the quantized [N, K] weight."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    r = 0 if A is None else A.shape[0]
    if A is not None:
        _need(A, "A", torch.bfloat16, r * K)
        _need(B, "B", torch.bfloat16, N * r)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if y is None else y
    _need(y, "y", torch.bfloat16, M * N)
    ws = nf4_lora_linear_workspace_size(M, r)
    if workspace is None and ws > 0:
        workspace = torch.empty(ws, dtype=torch.uint8, device=x.device)
    st = lib().nf4_lora_linear_fwd(_p(x), M, K, N, _p(packed), _p(absmax_q), _p(absmax2), _p(offset), _p(A), _p(B),
                                   r, float(scaling), _p(y), _p(workspace),
                                   0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _stream(stream))
    _check("nf4_lora_linear_fwd", st)
    return y


NOALLOC_SCRATCH_BYTES = 4 * 1024 * 1024


def nf4_lora_linear_fwd_noalloc(x: torch.Tensor, packed: torch.Tensor, absmax_q: Optional[torch.Tensor],
                                absmax2: torch.Tensor, offset: Optional[torch.Tensor], N: int,
                                A: Optional[torch.Tensor] = None, B: Optional[torch.Tensor] = None,
                                scaling: float = 1.0, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """nf4_lora_linear_fwd without a workspace, for callers that cannot
    allocate device memory: the low-rank intermediate uses the library's
    fixed 4 MiB device scratch.  Pass a preallocated ``y`` to allocate nothing
    here either.  Calls that may overlap on the GPU race on the scratch."""
    _need(x, "x", torch.bfloat16)
    M, K = x.shape
    r = 0 if A is None else A.shape[0]
    if A is not None:
        _need(A, "A", torch.bfloat16, r * K)
        _need(B, "B", torch.bfloat16, N * r)
    y = torch.empty(M, N, dtype=torch.bfloat16, device=x.device) if y is None else y
    _need(y, "y", torch.bfloat16, M * N)
    st = lib().nf4_lora_linear_fwd_noalloc(_p(x), M, K, N, _p(packed), _p(absmax_q), _p(absmax2), _p(offset),
                                           _p(A), _p(B), r, float(scaling), _p(y), _stream(stream))
    _check("nf4_lora_linear_fwd_noalloc", st)
    return y


def nf4_device_status(stream=None) -> int:
    """Synchronize the stream; raise Nf4Error if a kernel's bounded wait expired."""
    st = lib().nf4_device_status(_stream(stream))
    _check("nf4_device_status", st)
    return st


def nf4_lora_linear_bwd_workspace_size(M: int, N: int, K: int, r: int) -> int:
    return int(lib().nf4_lora_linear_bwd_workspace_size(M, N, K, r))


def nf4_lora_linear_bwd(g: torch.Tensor, x: Optional[torch.Tensor], packed: torch.Tensor,
                        absmax_q: Optional[torch.Tensor], absmax2: torch.Tensor, offset: Optional[torch.Tensor],
                        K: int, A: Optional[torch.Tensor] = None, B: Optional[torch.Tensor] = None,
                        scaling: float = 1.0, want=("dx", "dA", "dB"), dx: Optional[torch.Tensor] = None,
                        dA: Optional[torch.Tensor] = None, dB: Optional[torch.Tensor] = None,
                        workspace: Optional[torch.Tensor] = None, stream=None):
    """Backward of nf4_lora_linear_fwd: returns (dx bf16 [M, K], dA fp32 [r, K],
    dB fp32 [N, r]), None for an output not in `want` (or without an adapter)."""
    M, N = g.shape
    _need(g, "g", torch.bfloat16)
    r = 0
    if A is not None and B is not None:
        r = A.shape[0]
        _need(A, "A", torch.bfloat16, r * K)
        _need(B, "B", torch.bfloat16, N * r)
    if "dx" in want:
        if dx is None:
            dx = torch.empty(M, K, dtype=torch.bfloat16, device=g.device)
        _need(dx, "dx", torch.bfloat16, M * K)
    else:
        dx = None
    if r > 0 and "dA" in want:
        if dA is None:
            dA = torch.empty(r, K, dtype=torch.float32, device=g.device)
        _need(dA, "dA", torch.float32, r * K)
    else:
        dA = None
    if r > 0 and "dB" in want:
        if dB is None:
            dB = torch.empty(N, r, dtype=torch.float32, device=g.device)
        _need(dB, "dB", torch.float32, N * r)
    else:
        dB = None
    if x is not None:
        _need(x, "x", torch.bfloat16, M * K)
    ws_bytes = nf4_lora_linear_bwd_workspace_size(M, N, K, r)
    if workspace is None and ws_bytes > 0:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=g.device)
    st = lib().nf4_lora_linear_bwd(_p(g), _p(x), M, K, N, _p(packed), _p(absmax_q), _p(absmax2), _p(offset), _p(A),
                                   _p(B), r, float(scaling), _p(dx), _p(dA), _p(dB), _p(workspace),
                                   0 if workspace is None else workspace.numel(), _stream(stream))
    _check("nf4_lora_linear_bwd", st)
    return dx, dA, dB


def nf4_merge_requantize(packed: torch.Tensor, absmax_q: Optional[torch.Tensor], absmax2: torch.Tensor,
                         offset: Optional[torch.Tensor], N: int, K: int, A: Optional[torch.Tensor] = None,
                         B: Optional[torch.Tensor] = None, scaling: float = 1.0,
                         packed_out: Optional[torch.Tensor] = None, absmax_out: Optional[torch.Tensor] = None,
                         stream=None):
    """W' = fma(scaling, B A, dequant(W)) quantized again; returns (packed_out
    uint8 [N K / 2], absmax_out fp32 [N K / 64])."""
    n = N * K
    _need(packed, "packed", torch.uint8, n // 2)
    if absmax_q is not None:
        _need(absmax_q, "absmax_q", torch.uint8, n // BLOCKSIZE)
    _need(absmax2, "absmax2", torch.float32)
    r = 0
    if A is not None and B is not None:
        r = A.shape[0]
        _need(A, "A", torch.bfloat16, r * K)
        _need(B, "B", torch.bfloat16, N * r)
    if packed_out is None:
        packed_out = torch.empty(n // 2, dtype=torch.uint8, device=packed.device)
    if absmax_out is None:
        absmax_out = torch.empty(n // BLOCKSIZE, dtype=torch.float32, device=packed.device)
    _need(packed_out, "packed_out", torch.uint8, n // 2)
    _need(absmax_out, "absmax_out", torch.float32, n // BLOCKSIZE)
    st = lib().nf4_merge_requantize(_p(packed), _p(absmax_q), _p(absmax2), _p(offset), N, K, _p(A), _p(B), r,
                                    float(scaling), _p(packed_out), _p(absmax_out), _stream(stream))
    _check("nf4_merge_requantize", st)
    return packed_out, absmax_out


def nf4_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launch the bounded-wait check (a wait that expires after limit_ns);
    the next nf4_device_status() raises Nf4Error with NF4_ERR_TIMEOUT."""
    _check("nf4_selftest_wait_timeout", lib().nf4_selftest_wait_timeout(int(limit_ns), _stream(stream)))


@dataclass
class QuantState:
    """The quantized form of one weight W[N, K] (flattened row-major)."""
    packed: torch.Tensor
    absmax_q: Optional[torch.Tensor]
    absmax2: torch.Tensor
    offset: Optional[torch.Tensor]
    shape: tuple

    @property
    def numel(self) -> int:
        return self.shape[0] * self.shape[1]

    def nbytes(self) -> int:
        t = [self.packed, self.absmax_q, self.absmax2, self.offset]
        return sum(x.numel() * x.element_size() for x in t if x is not None)


def merge_and_requantize(state: "QuantState", A: torch.Tensor, B: torch.Tensor, scaling: float,
                         double_quant: bool = True, centre: bool = True, stream=None) -> "QuantState":
    """nf4_merge_requantize followed (optionally) by nf4_double_quantize: the
    adapter merged into the quantized base, in the stored format again."""
    N, K = state.shape
    packed, absmax = nf4_merge_requantize(state.packed, state.absmax_q, state.absmax2, state.offset, N, K, A, B,
                                          scaling, stream=stream)
    if not double_quant:
        return QuantState(packed, None, absmax, None, (N, K))
    q8, c2, off = nf4_double_quantize(absmax, centre=centre, stream=stream)
    return QuantState(packed, q8, c2, off, (N, K))


def quantize_weight(w: torch.Tensor, double_quant: bool = True, centre: bool = True, stream=None) -> QuantState:
    """nf4_quantize followed (optionally) by nf4_double_quantize."""
    packed, absmax = nf4_quantize(w.reshape(-1), stream=stream)
    if not double_quant:
        return QuantState(packed, None, absmax, None, tuple(w.shape))
    q8, c2, off = nf4_double_quantize(absmax, centre=centre, stream=stream)
    return QuantState(packed, q8, c2, off, tuple(w.shape))
