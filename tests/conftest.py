"""Shared test configuration.

Markers: ``gpu`` marks tests that need a CUDA device (the parity tests of the
CUDA library against the CPU oracle).  ``python -m pytest -m "not gpu"`` runs
the oracle pins, host logic and C-ABI symbol checks on a machine without a GPU.
"""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.lib()
    return oracle


def read_golden_values(name):
    vals = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                vals.append(line)
    return vals


def read_golden_kv(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                k, v = line.split("=")
                out[k.strip()] = float(v)
    return out


@pytest.fixture(scope="session")
def nf4lib():
    """The CUDA library, built in-tree for sm_100a (nvcc cross-compiles on a
    machine without a GPU as well)."""
    from qlora_nf4_quantize_b200 import build as b
    b.build()
    import qlora_nf4_quantize_b200 as q
    q.lib()
    return q


@pytest.fixture(scope="session")
def cuda_device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("gpu test needs a CUDA device")
    return torch.device("cuda:0")


def rel_error_stats(y, ref):
    """Max and mean relative error with the denominator floored at 1e-2 of
    the reference's rms (so outputs near zero are judged on an absolute
    scale), plus the Frobenius relative error."""
    import numpy as np
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    den = np.maximum(np.abs(ref), 1e-2 * rms)
    rel = np.abs(y - ref) / den
    fro = float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))
    return float(rel.max()) if rel.size else 0.0, float(rel.mean()) if rel.size else 0.0, fro


MATMUL_MAX_REL = 1e-2
MATMUL_MEAN_REL = 2e-3


# ---------------------------------------------------------------- output guards
# compute-sanitizer is not available where the GPU tests run, so every output
# buffer of a GPU parity test sits between two poisoned guard regions: a write
# past either end of the buffer changes a guard byte and fails the test.
GUARD_BYTES = 4096
GUARD_FILL = 0xA5


def guarded(shape, dtype, device, fill=None):
    """A tensor of `shape` and `dtype` on `device` placed between two
    GUARD_BYTES regions filled with GUARD_FILL (16-byte alignment kept).
    ``fill`` sets the tensor's own contents (default: the poison bytes too,
    so an output element the call forgets to write also shows up as a
    mismatch).  check_guards() verifies the guards after the call."""
    import math

    import torch
    shape = (shape,) if isinstance(shape, int) else tuple(shape)
    n = math.prod(shape)
    nbytes = n * torch.empty(0, dtype=dtype).element_size()
    raw = torch.full((2 * GUARD_BYTES + nbytes,), GUARD_FILL, dtype=torch.uint8, device=device)
    t = raw[GUARD_BYTES:GUARD_BYTES + nbytes].view(dtype).view(shape)
    if fill is not None:
        t.fill_(fill)
    t._nf4_guard = (raw, nbytes)
    return t


def check_guards(*tensors):
    """Assert the guard regions around each guarded() tensor are intact."""
    import torch
    for i, t in enumerate(tensors):
        if t is None:
            continue
        raw, nbytes = t._nf4_guard
        head = raw[:GUARD_BYTES]
        tail = raw[GUARD_BYTES + nbytes:]
        bad_head = torch.nonzero(head != GUARD_FILL)
        bad_tail = torch.nonzero(tail != GUARD_FILL)
        assert bad_head.numel() == 0, f"buffer {i}: write before its start at byte {int(bad_head[-1]) - GUARD_BYTES}"
        assert bad_tail.numel() == 0, f"buffer {i}: write past its end at byte +{int(bad_tail[0])}"
