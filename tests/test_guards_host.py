"""The output guards of the GPU parity tests (conftest.guarded /
check_guards), checked on the CPU: a write one byte before a guarded buffer
or one byte past its end is reported, an untouched buffer passes, and the
buffer keeps 16-byte alignment for the library's pointer checks."""
import pytest
import torch

from conftest import GUARD_BYTES, check_guards, guarded


@pytest.mark.parametrize("shape,dtype", [((3, 5), torch.bfloat16), (7, torch.uint8), ((2, 9), torch.float32),
                                         (0, torch.float32)])
def test_guards_catch_writes_outside_the_buffer(shape, dtype):
    t = guarded(shape, dtype, "cpu", fill=0)
    assert t.data_ptr() % 16 == 0
    check_guards(t)
    raw, nbytes = t._nf4_guard
    raw[GUARD_BYTES - 1] = 0
    with pytest.raises(AssertionError, match="before its start"):
        check_guards(t)
    raw[GUARD_BYTES - 1] = 0xA5
    raw[GUARD_BYTES + nbytes] = 0
    with pytest.raises(AssertionError, match="past its end"):
        check_guards(t)


def test_default_fill_is_the_poison():
    t = guarded(4, torch.uint8, "cpu")
    assert torch.all(t == 0xA5)
