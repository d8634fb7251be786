"""CPU oracle for NF4 quantization, double quantization, dequantization and the
frozen-base LoRA linear.

TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and the
benchmark's CPU-baseline leg use this module; the product path never imports
it.  The arithmetic lives in ``nf4_oracle.c`` (plain C, strict IEEE, fp64
sums), which shares no code with the CUDA library.  This wrapper only builds
that file with gcc, loads it with ctypes and marshals numpy arrays.

Parity status of each function (what pins it) is stated in the docstrings;
the conventions that no page fixes (nibble order, tie rule, centring mean and
its summation order) are "parity unpinned" against the pages and are pinned
only oracle-vs-GPU.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "nf4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_nf4.so")
_lock = threading.Lock()
_lib = None

BLOCKSIZE = 64
DQ_BLOCKSIZE = 256


def build(force: bool = False) -> str:
    """Compile nf4_oracle.c into liboracle_nf4.so beside it (strict IEEE flags)."""
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i64 = ctypes.c_int64
            L.nf4o_codebook.argtypes = [P]
            L.nf4o_norm_ppf.argtypes = [ctypes.c_double]
            L.nf4o_norm_ppf.restype = ctypes.c_double
            L.nf4o_codebook_construct.argtypes = [ctypes.c_double, P]
            L.nf4o_bf16_to_f32.argtypes = [ctypes.c_uint16]
            L.nf4o_bf16_to_f32.restype = ctypes.c_float
            L.nf4o_f32_to_bf16.argtypes = [ctypes.c_float]
            L.nf4o_f32_to_bf16.restype = ctypes.c_uint16
            L.nf4o_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.nf4o_e4m3_decode.restype = ctypes.c_double
            L.nf4o_e4m3_encode.argtypes = [ctypes.c_float]
            L.nf4o_e4m3_encode.restype = ctypes.c_uint8
            L.nf4o_code_of.argtypes = [ctypes.c_float]
            L.nf4o_code_of.restype = ctypes.c_int
            L.nf4o_quantize_f32.argtypes = [P, i64, ctypes.c_int, P, P]
            L.nf4o_quantize_bf16.argtypes = [P, i64, ctypes.c_int, P, P]
            L.nf4o_dq_mean.argtypes = [P, i64, ctypes.c_int]
            L.nf4o_dq_mean.restype = ctypes.c_float
            L.nf4o_double_quantize.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P, P]
            L.nf4o_dq_run_sums.argtypes = [P, i64, ctypes.c_int, P]
            L.nf4o_dq_mean_from_run_sums.argtypes = [P, i64, i64]
            L.nf4o_dq_mean_from_run_sums.restype = ctypes.c_float
            L.nf4o_double_quantize_with_mean.argtypes = [P, i64, ctypes.c_int, ctypes.c_float, P, P]
            L.nf4o_dequantize_f32.argtypes = [P, P, P, P, i64, ctypes.c_int, ctypes.c_int, P]
            L.nf4o_dequantize_bf16.argtypes = [P, P, P, P, i64, ctypes.c_int, ctypes.c_int, P]
            L.nf4o_lora_linear.argtypes = [P, i64, i64, i64, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                           P, P, ctypes.c_int, ctypes.c_float, P, i64, P]
            L.nf4o_lora_linear_bwd.argtypes = [P, P, i64, i64, i64, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                               P, P, ctypes.c_int, ctypes.c_float, P, i64, P, P, P]
            L.nf4o_merge_weight.argtypes = [P, P, P, P, i64, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int,
                                            ctypes.c_float, i64, i64, P]
            L.nf4o_merge_requantize.argtypes = [P, P, P, P, i64, ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int,
                                                ctypes.c_float, i64, i64, P, P]
            L.nf4o_e4m3_encode_array.argtypes = [P, i64, P]
            L.nf4o_f32_to_bf16_array.argtypes = [P, i64, P]
            L.nf4o_code_of_array.argtypes = [P, i64, P]
            _lib = L
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- codebook
def codebook() -> np.ndarray:
    """The sixteen NF4 levels as printed on the Mathematical Foundations page
    (section "4-Bit NormalFloat (NF4)"), float32.  Pinned to the golden copy
    of the printed table and to the quantile construction."""
    out = np.empty(16, np.float32)
    lib().nf4o_codebook(_ptr(out))
    return out


def norm_ppf(p: float) -> float:
    """Inverse standard normal CDF by bisection on erfc.  Pinned to
    scipy.special.ndtri (library routine) and closed-form quantiles."""
    return lib().nf4o_norm_ppf(float(p))


def codebook_construct(delta: float) -> np.ndarray:
    """Quantile construction of the levels (7 negative, zero, 8 positive,
    normalised to +-1) with outermost probability ``delta``; float64."""
    out = np.empty(16, np.float64)
    lib().nf4o_codebook_construct(float(delta), _ptr(out))
    return out


# ---------------------------------------------------------------- scalar formats
def bf16_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(f: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even."""
    f = np.ascontiguousarray(f, np.float32).ravel()
    out = np.empty(f.size, np.uint16)
    lib().nf4o_f32_to_bf16_array(_ptr(f), f.size, _ptr(out))
    return out


def e4m3_decode(c: int) -> float:
    return lib().nf4o_e4m3_decode(int(c))


def e4m3_encode(y: float) -> int:
    return int(lib().nf4o_e4m3_encode(float(np.float32(y))))


def e4m3_encode_array(y: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y, np.float32).ravel()
    out = np.empty(y.size, np.uint8)
    lib().nf4o_e4m3_encode_array(_ptr(y), y.size, _ptr(out))
    return out


def code_of(x: float) -> int:
    """Nearest-level index of a float32 value (lower index on ties)."""
    return int(lib().nf4o_code_of(float(np.float32(x))))


def code_of_array(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, np.float32).ravel()
    out = np.empty(x.size, np.uint8)
    lib().nf4o_code_of_array(_ptr(x), x.size, _ptr(out))
    return out


# ---------------------------------------------------------------- quantization
def quantize(w: np.ndarray, blocksize: int = BLOCKSIZE):
    """Blockwise NF4 quantization of a flattened tensor.

    ``w``: float32 array, or uint16 array holding bfloat16 bit patterns.
    Returns (packed uint8[n/2], absmax float32[ceil(n/blocksize)])."""
    w = np.ascontiguousarray(w).ravel()
    n = w.size
    if n % 2:
        raise ValueError("n must be even")
    nb = (n + blocksize - 1) // blocksize
    packed = np.zeros(n // 2, np.uint8)
    absmax = np.zeros(nb, np.float32)
    if w.dtype == np.float32:
        lib().nf4o_quantize_f32(_ptr(w), n, blocksize, _ptr(packed), _ptr(absmax))
    elif w.dtype == np.uint16:
        lib().nf4o_quantize_bf16(_ptr(w), n, blocksize, _ptr(packed), _ptr(absmax))
    else:
        raise TypeError("w must be float32 or uint16 (bf16 bits)")
    return packed, absmax


def dq_mean(absmax: np.ndarray, dq_blocksize: int = DQ_BLOCKSIZE) -> np.float32:
    a = np.ascontiguousarray(absmax, np.float32)
    return np.float32(lib().nf4o_dq_mean(_ptr(a), a.size, dq_blocksize))


def double_quantize(absmax: np.ndarray, dq_blocksize: int = DQ_BLOCKSIZE, centre: bool = True):
    """Returns (codes uint8[nb], absmax2 float32[nd], offset float32)."""
    a = np.ascontiguousarray(absmax, np.float32)
    nb = a.size
    nd = (nb + dq_blocksize - 1) // dq_blocksize
    codes = np.zeros(nb, np.uint8)
    absmax2 = np.zeros(nd, np.float32)
    off = np.zeros(1, np.float32)
    lib().nf4o_double_quantize(_ptr(a), nb, dq_blocksize, 1 if centre else 0,
                               _ptr(codes), _ptr(absmax2), _ptr(off))
    return codes, absmax2, np.float32(off[0])


def dq_run_sums(absmax: np.ndarray, dq_blocksize: int = DQ_BLOCKSIZE) -> np.ndarray:
    """Step 1 of the mean: the sequential binary64 sum of each run."""
    a = np.ascontiguousarray(absmax, np.float32)
    out = np.zeros(-(-a.size // dq_blocksize), np.float64)
    lib().nf4o_dq_run_sums(_ptr(a), a.size, dq_blocksize, _ptr(out))
    return out


def dq_mean_from_run_sums(run_sums: np.ndarray, nblocks: int) -> np.float32:
    """Steps 2 and 3 of the mean (pairwise tree, division, rounding) on the
    run sums of a whole tensor of nblocks constants."""
    s = np.ascontiguousarray(run_sums, np.float64)
    return np.float32(lib().nf4o_dq_mean_from_run_sums(_ptr(s), s.size, int(nblocks)))


def double_quantize_with_mean(absmax: np.ndarray, mu, dq_blocksize: int = DQ_BLOCKSIZE):
    """Double quantization of the runs of ``absmax`` with a given mean mu;
    returns (codes uint8[nb], absmax2 float32[nd])."""
    a = np.ascontiguousarray(absmax, np.float32)
    codes = np.zeros(a.size, np.uint8)
    absmax2 = np.zeros(-(-a.size // dq_blocksize), np.float32)
    lib().nf4o_double_quantize_with_mean(_ptr(a), a.size, dq_blocksize, float(mu), _ptr(codes), _ptr(absmax2))
    return codes, absmax2


def dequantize(packed, codes, scales, offset, n, out_dtype="f32",
               blocksize: int = BLOCKSIZE, dq_blocksize: int = DQ_BLOCKSIZE):
    """Dequantize.  ``codes`` None means ``scales`` are the fp32 first-level
    constants (no double quantization); otherwise ``scales`` are c2 and
    ``offset`` the mean (None for no centring).  out_dtype 'f32' gives
    float32, 'bf16' gives uint16 bf16 bit patterns."""
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.float32)
    codes = None if codes is None else np.ascontiguousarray(codes, np.uint8)
    off = None if offset is None else np.array([offset], np.float32)
    if out_dtype == "f32":
        out = np.empty(n, np.float32)
        lib().nf4o_dequantize_f32(_ptr(packed), _ptr(codes), _ptr(scales), _ptr(off), n,
                                  blocksize, dq_blocksize, _ptr(out))
    elif out_dtype == "bf16":
        out = np.empty(n, np.uint16)
        lib().nf4o_dequantize_bf16(_ptr(packed), _ptr(codes), _ptr(scales), _ptr(off), n,
                                   blocksize, dq_blocksize, _ptr(out))
    else:
        raise ValueError(out_dtype)
    return out


def lora_linear(x_bf16, K, N, packed, codes, scales, offset, A_bf16, B_bf16, r, s,
                rows=None, blocksize: int = BLOCKSIZE, dq_blocksize: int = DQ_BLOCKSIZE):
    """y[rows, :] in float64 for y = x deq(W)^T + s (x A^T) B^T (bf16 inputs as
    uint16 bit patterns, x [M, K], W [N, K] quantized, A [r, K], B [N, r])."""
    x = np.ascontiguousarray(x_bf16, np.uint16).reshape(-1, K)
    M = x.shape[0]
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    y = np.empty((rows.size, N), np.float64)
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.float32)
    codes = None if codes is None else np.ascontiguousarray(codes, np.uint8)
    off = None if offset is None else np.array([offset], np.float32)
    A = None if A_bf16 is None else np.ascontiguousarray(A_bf16, np.uint16)
    B = None if B_bf16 is None else np.ascontiguousarray(B_bf16, np.uint16)
    lib().nf4o_lora_linear(_ptr(x), M, K, N, _ptr(packed), _ptr(codes), _ptr(scales), _ptr(off),
                           blocksize, dq_blocksize, _ptr(A), _ptr(B), int(r if A is not None else 0),
                           float(s), _ptr(rows), rows.size, _ptr(y))
    return y


def _merge_args(packed, codes, scales, offset, K, A_bf16, B_bf16, r):
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.float32)
    codes = None if codes is None else np.ascontiguousarray(codes, np.uint8)
    off = None if offset is None else np.array([offset], np.float32)
    N = packed.size * 2 // K
    if r == 0:  # no adapter: W' = w~
        return packed, codes, scales, off, np.zeros(1, np.uint16), np.zeros(1, np.uint16), N
    A = np.ascontiguousarray(A_bf16, np.uint16).reshape(r, K)
    B = np.ascontiguousarray(B_bf16, np.uint16).reshape(N, r)
    return packed, codes, scales, off, A, B, N


def merge_weight(packed, codes, scales, offset, K, A_bf16, B_bf16, r, s, row0=0, nrows=None,
                 blocksize: int = BLOCKSIZE, dq_blocksize: int = DQ_BLOCKSIZE):
    """W' = fma(s, d, w~) with d the fixed-order binary32 fma chain of
    B[n, :] A[:, k] (the merge reading of nf4o_merge_weight), rows
    [row0, row0 + nrows) of W[N, K]; float32 [nrows, K].
    Pinned by the delta against an fp64 matmul, the s = 0 identity, and an
    exact-rational re-evaluation of the chain on a tiny case."""
    packed, codes, scales, off, A, B, N = _merge_args(packed, codes, scales, offset, K, A_bf16, B_bf16, r)
    nrows = N - row0 if nrows is None else nrows
    out = np.empty((nrows, K), np.float32)
    lib().nf4o_merge_weight(_ptr(packed), _ptr(codes), _ptr(scales), _ptr(off), int(K), blocksize, dq_blocksize,
                            _ptr(A), _ptr(B), int(r), float(s), int(row0), int(nrows), _ptr(out))
    return out


def merge_requantize(packed, codes, scales, offset, K, A_bf16, B_bf16, r, s, row0=0, nrows=None,
                     blocksize: int = BLOCKSIZE, dq_blocksize: int = DQ_BLOCKSIZE):
    """merge_weight's rows quantized again (blockwise NF4, fp32 constants):
    (packed uint8 [nrows K / 2], absmax float32 [nrows K / 64])."""
    packed, codes, scales, off, A, B, N = _merge_args(packed, codes, scales, offset, K, A_bf16, B_bf16, r)
    nrows = N - row0 if nrows is None else nrows
    pk = np.empty(nrows * K // 2, np.uint8)
    ab = np.empty(nrows * K // blocksize, np.float32)
    lib().nf4o_merge_requantize(_ptr(packed), _ptr(codes), _ptr(scales), _ptr(off), int(K), blocksize,
                                dq_blocksize, _ptr(A), _ptr(B), int(r), float(s), int(row0), int(nrows), _ptr(pk),
                                _ptr(ab))
    return pk, ab


def lora_linear_bwd(g_bf16, x_bf16, K, N, packed, codes, scales, offset, A_bf16, B_bf16, r, s, rows=None,
                    want=("dx", "dA", "dB"), blocksize: int = BLOCKSIZE, dq_blocksize: int = DQ_BLOCKSIZE):
    """Backward of lora_linear (the adjoint of the forward in the frozen
    weight's layout): returns a dict with float64 'dx' [len(rows), K],
    'dA' [r, K], 'dB' [N, r] as requested (g = dL/dy, bf16 bit patterns
    [M, N]; x bf16 [M, K] needed for dA, dB).  Pinned by the adjoint
    identities <g, y(x)> = <dx, x>, <g, y_A(E)> = <dA, E>, <g, y_B(F)> =
    <dB, F> against the (separately pinned) forward."""
    g = np.ascontiguousarray(g_bf16, np.uint16).reshape(-1, N)
    M = g.shape[0]
    x = None if x_bf16 is None else np.ascontiguousarray(x_bf16, np.uint16).reshape(M, K)
    rows = np.arange(M, dtype=np.int64) if rows is None else np.ascontiguousarray(rows, np.int64)
    packed = np.ascontiguousarray(packed, np.uint8)
    scales = np.ascontiguousarray(scales, np.float32)
    codes = None if codes is None else np.ascontiguousarray(codes, np.uint8)
    off = None if offset is None else np.array([offset], np.float32)
    lora = A_bf16 is not None and B_bf16 is not None and r > 0
    A = np.ascontiguousarray(A_bf16, np.uint16) if lora else None
    B = np.ascontiguousarray(B_bf16, np.uint16) if lora else None
    out = {}
    dx = np.empty((rows.size, K), np.float64) if "dx" in want else None
    dA = np.empty((r, K), np.float64) if ("dA" in want and lora) else None
    dB = np.empty((N, r), np.float64) if ("dB" in want and lora) else None
    lib().nf4o_lora_linear_bwd(_ptr(g), _ptr(x), M, int(K), int(N), _ptr(packed), _ptr(codes), _ptr(scales),
                               _ptr(off), blocksize, dq_blocksize, _ptr(A), _ptr(B), int(r if lora else 0), float(s),
                               _ptr(rows), rows.size, _ptr(dx), _ptr(dA), _ptr(dB))
    for name, arr in (("dx", dx), ("dA", dA), ("dB", dB)):
        if arr is not None:
            out[name] = arr
    return out
