"""Compile-only checks (nvcc, no GPU) of the library's build option for
decode-size calls: NF4_SMALL_M_TC_FROM picks the token count from which
calls of up to 16 tokens take the split 16-token tensor-core pipeline
instead of the decode kernel (17, the default, sends all of them to the
decode kernel).  The dispatch that the option selects must keep compiling,
and values outside 9..17 must be refused at compile time (the decode kernel
serves at least 1..8 tokens and at most 16)."""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
from qlora_nf4_quantize_b200 import build  # noqa: E402

pytestmark = pytest.mark.skipif(not os.path.exists(build.NVCC), reason="nvcc not installed")


def compile_linear(tmp_path, value):
    src = os.path.join(build.CSRC, "linear.cu")
    out = str(tmp_path / f"linear_{value}.o")
    cmd = [build.NVCC, *build.ARCH, *build.FLAGS, f"-DNF4_SMALL_M_TC_FROM={value}", "-c", src, "-o", out]
    return subprocess.run(cmd, capture_output=True, text=True)


@pytest.mark.parametrize("value", [9, 13, 17])
def test_split_pipeline_routing_builds(tmp_path, value):
    r = compile_linear(tmp_path, value)
    assert r.returncode == 0, r.stderr


@pytest.mark.parametrize("value", [8, 18])
def test_routing_outside_the_decode_kernel_range_is_refused(tmp_path, value):
    r = compile_linear(tmp_path, value)
    assert r.returncode != 0
    assert "the decode kernel serves" in r.stderr + r.stdout
