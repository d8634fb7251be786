"""Host-side checks of the C ABI (no GPU needed): the library builds for
sm_100a, exports every entry point include/nf4.h declares, and rejects bad
arguments on the host before touching the device."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from conftest import ROOT


def declared_entry_points():
    with open(os.path.join(ROOT, "include", "nf4.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^NF4_API\s+[\w\s\*]+?\b(nf4_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_five_calls():
    names = declared_entry_points()
    for fn in ("nf4_codebook", "nf4_quantize", "nf4_double_quantize", "nf4_dequantize", "nf4_lora_linear_fwd"):
        assert fn in names


def test_library_exports_every_declared_symbol(nf4lib):
    out = subprocess.run(["nm", "-D", "--defined-only", nf4lib.nf4.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\bT\s+(nf4_\w+)", out))
    missing = [n for n in declared_entry_points() if n not in exported]
    assert not missing, missing
    L = nf4lib.lib()
    for n in declared_entry_points():
        assert hasattr(L, n)


def test_codebook_call_matches_oracle(nf4lib, oracle_mod):
    got = nf4lib.nf4_codebook().numpy()
    assert np.array_equal(got, oracle_mod.codebook())


def test_merge_arguments_checked_on_the_host(nf4lib):
    L = nf4lib.lib()
    fake = ctypes.c_void_p(0x1000)
    args = lambda N, K, r: (fake, fake, fake, fake, N, K, fake, fake, r, 1.0, fake, fake, None)
    assert L.nf4_merge_requantize(*args(8, 100, 16)) == 1   # K not a multiple of 64
    assert L.nf4_merge_requantize(*args(0, 128, 16)) == 1   # no rows
    assert L.nf4_merge_requantize(*args(8, 128, 65)) == 2   # rank above 64
    assert L.nf4_merge_requantize(*args(8, 128, -1)) == 1
    bad = ctypes.c_void_p(0x1004)                            # misaligned output
    assert L.nf4_merge_requantize(fake, fake, fake, fake, 8, 128, fake, fake, 16, 1.0, bad, fake, None) == 1


def test_selftest_limit_checked_on_the_host(nf4lib):
    L = nf4lib.lib()
    for bad in (0, -5, 1000000001):
        assert L.nf4_selftest_wait_timeout(bad, None) == 1  # NF4_ERR_INVALID, nothing launched


def test_host_validation_before_any_device_work(nf4lib):
    L = nf4lib.lib()
    fake = ctypes.c_void_p(0x1000)  # never dereferenced: validation fails first
    # block sizes other than 64 / 256
    assert L.nf4_quantize(fake, 0, 128, 32, fake, fake, None) == 2
    assert L.nf4_double_quantize(fake, 4, 128, fake, fake, None, None, 0, None) == 2
    assert L.nf4_dequantize(fake, fake, fake, None, 128, 64, 128, fake, 0, None) == 2
    # odd n, negative n, NULL pointers, misaligned pointers
    assert L.nf4_quantize(fake, 0, 127, 64, fake, fake, None) == 1
    assert L.nf4_quantize(fake, 0, -2, 64, fake, fake, None) == 1
    assert L.nf4_quantize(None, 0, 128, 64, fake, fake, None) == 1
    assert L.nf4_quantize(ctypes.c_void_p(0x1004), 0, 128, 64, fake, fake, None) == 1
    assert L.nf4_dequantize(fake, None, fake, fake, 128, 64, 256, fake, 0, None) == 1  # offset without codes
    # empty inputs are a no-op success
    assert L.nf4_quantize(None, 0, 0, 64, None, None, None) == 0
    assert L.nf4_double_quantize(None, 0, 256, None, None, None, None, 0, None) == 0
    # linear: unsupported rank, K not a multiple of 64, missing workspace
    assert L.nf4_lora_linear_fwd(fake, 4, 128, 64, fake, fake, fake, fake, fake, fake, 8, 1.0, fake, fake, 1 << 20, None) == 2
    assert L.nf4_lora_linear_fwd(fake, 4, 100, 64, fake, fake, fake, fake, None, None, 0, 1.0, fake, None, 0, None) == 1
    assert L.nf4_lora_linear_fwd(fake, 4, 128, 64, fake, fake, fake, fake, fake, fake, 16, 1.0, fake, None, 0, None) == 1
    assert L.nf4_status_string(4) == b"NF4_ERR_TIMEOUT"


def test_workspace_sizes(nf4lib):
    assert nf4lib.nf4_double_quantize_workspace_size(0) == 0
    # fp64 run sums, then the chunk sums (32 runs each)
    assert nf4lib.nf4_double_quantize_workspace_size(2048) == (8 + 1) * 8        # 8 runs, 1 chunk
    assert nf4lib.nf4_double_quantize_workspace_size(256 * 33) == (33 + 2) * 8   # 33 runs, 2 chunks
    # quantize + DQ in one call: fp32 constants (256-byte aligned), then the same sums
    assert nf4lib.nf4_quantize_dq_workspace_size(4096 * 4096) == 262144 * 4 + (1024 + 32) * 8
    assert nf4lib.nf4_quantize_dq_workspace_size(130) == 256 + (1 + 1) * 8
    assert nf4lib.nf4_quantize_dq_workspace_size(128, 32, 256) == 0
    # [t_hi | t_lo | pad] rows of round_up(2r, 64) bf16; nothing without an
    # adapter (decode-size calls need no scratch of their own)
    assert nf4lib.nf4_lora_linear_workspace_size(16, 16) == 16 * 64 * 2
    assert nf4lib.nf4_lora_linear_workspace_size(3, 16) == 3 * 64 * 2
    assert nf4lib.nf4_lora_linear_workspace_size(9, 64) == 9 * 128 * 2
    assert nf4lib.nf4_lora_linear_workspace_size(16, 0) == 0
    assert nf4lib.nf4_lora_linear_workspace_size(1, 0) == 0
    assert nf4lib.nf4_lora_linear_workspace_size(17, 0) == 0
    assert nf4lib.nf4_lora_linear_workspace_size(4096, 0) == 0
    assert nf4lib.nf4_lora_linear_workspace_size(4096, 64) == 4096 * 128 * 2


def test_sharded_dq_arguments_checked_on_the_host(nf4lib):
    L = nf4lib.lib()
    fake = ctypes.c_void_p(0x1000)
    assert L.nf4_dq_run_sums(fake, 512, 128, fake, None) == 2            # second-level block must be 256
    assert L.nf4_dq_run_sums(fake, -1, 256, fake, None) == 1
    assert L.nf4_dq_run_sums(None, 0, 256, None, None) == 0               # empty: no-op
    assert L.nf4_dq_run_sums(fake, 512, 256, ctypes.c_void_p(0x1008), None) == 1  # misaligned sums
    ws = 1 << 20
    args = lambda nb, tot, off: (fake, nb, 256, fake, tot, fake, fake, off, fake, ws, None)
    assert L.nf4_double_quantize_sharded(*args(600, 500, fake)) == 1     # shard larger than the tensor
    assert L.nf4_double_quantize_sharded(*args(100, 500, None)) == 1     # the mean must be written
    assert L.nf4_double_quantize_sharded(*args(100, 0, fake)) == 1
    assert L.nf4_double_quantize_sharded(fake, 100, 256, fake, 500, fake, fake, fake, fake, 0, None) == 1
    assert nf4lib.lib().nf4_double_quantize_sharded_workspace_size(256 * 33, 256) == 16  # 2 chunk sums
