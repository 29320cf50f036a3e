"""Argument checks of attn_jvp_rope on the host (no GPU): every call here fails
validation before any device call, so the fake pointers are never used."""
import ctypes

import pytest

from attention_jvp_attn_b200 import _abi

FAKE = [0x10000 * (i + 1) for i in range(10)]  # q k tq tk cos sin q' k' tq' tk'


@pytest.fixture(scope="module")
def lib():
    from attention_jvp_attn_b200 import build
    build.build()
    return _abi.load()


def _rope(lib, shape, ptrs):
    sp = ctypes.byref(shape) if shape is not None else None
    return lib.attn_jvp_rope(sp, *ptrs, None)


def test_rejects_bad_shapes(lib):
    assert _rope(lib, None, FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _rope(lib, _abi.Shape(0, 8, 2, 64, 0, 0.0), FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _rope(lib, _abi.Shape(1, 0, 2, 64, 0, 0.0), FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _rope(lib, _abi.Shape(1, 8, 2, 32, 0, 0.0), FAKE) == _abi.ERR_UNSUPPORTED
    assert _rope(lib, _abi.Shape(1, 8, 2, 64, 7, 0.0), FAKE) == _abi.ERR_UNSUPPORTED


@pytest.mark.parametrize("i", range(10))
def test_rejects_null_and_misaligned_pointers(lib, i):
    s = _abi.Shape(1, 8, 2, 64, 0, 0.0)
    ptrs = list(FAKE)
    ptrs[i] = None
    assert _rope(lib, s, ptrs) == _abi.ERR_INVALID_ARGUMENT
    ptrs = list(FAKE)
    ptrs[i] += 4
    assert _rope(lib, s, ptrs) == _abi.ERR_MISALIGNED
