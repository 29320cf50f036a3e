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


# attn_jvp_fwd_rope: q k v tq tk tv cos sin, then q' k' tq' tk' o to lse
FUSED = [0x10000 * (i + 1) for i in range(15)]


def _fused(lib, shape, mask, ptrs):
    return lib.attn_jvp_fwd_rope(ctypes.byref(shape), *ptrs[:8], mask, *ptrs[8:], None)


def test_fused_checks_pointers(lib):
    s = _abi.Shape(1, 64, 2, 64, _abi.DTYPE_BF16, 0.0)
    m = _abi.Mask(0, 16, 2)  # teacher forcing, 2 chunks of 16: L = 64
    for i in range(15):
        ptrs = list(FUSED)
        ptrs[i] = None
        assert _fused(lib, s, m, ptrs) == _abi.ERR_INVALID_ARGUMENT
        ptrs = list(FUSED)
        ptrs[i] += 8
        assert _fused(lib, s, m, ptrs) == _abi.ERR_MISALIGNED


def test_fused_rejects_more_than_2_32_vectors(lib):
    # the rotation counts the four tensors' 16-byte vectors in 32 bits:
    # B L H d / 2 must stay below 2^32
    m = _abi.Mask(0, 1 << 14, 32)  # L = 2^20
    at = _abi.Shape(1, 1 << 20, 64, 128, _abi.DTYPE_BF16, 0.0)  # 2^26 rows x 64 = 2^32
    assert _fused(lib, at, m, FUSED) == _abi.ERR_UNSUPPORTED
