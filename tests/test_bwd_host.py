"""Argument checks of the backward entry points attn_jvp_bwd and
attn_jvp_bwd_groups on the host (no GPU): every call here fails validation
before any device call, so the fake pointers are never dereferenced."""
import ctypes

import pytest

from attention_jvp_attn_b200 import _abi

TF, BC = 0, 1
FAKE = [0x10000 * (i + 1) for i in range(10)]  # q k v o do lse dlse dq dk dv


@pytest.fixture(scope="module")
def lib():
    from attention_jvp_attn_b200 import build
    build.build()
    return _abi.load()


def _bwd(lib, shape, mask, ptrs):
    q, k, v, o, do, lse, dlse, dq, dk, dv = ptrs
    sp = ctypes.byref(shape) if shape is not None else None
    return lib.attn_jvp_bwd(sp, q, k, v, o, do, lse, dlse, mask, dq, dk, dv, None)


def _bwd_groups(lib, shape, groups, n, ptrs):
    q, k, v, o, do, lse, dlse, dq, dk, dv = ptrs
    arr = _abi.group_array(groups) if groups else None
    return lib.attn_jvp_bwd_groups(ctypes.byref(shape), q, k, v, o, do, lse, dlse, arr,
                                   len(groups) if n is None else n, dq, dk, dv, None)


def test_rejects_bad_shapes(lib):
    m = _abi.Mask(TF, 16, 4)
    assert _bwd(lib, None, m, FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _bwd(lib, _abi.Shape(1, 127, 2, 64, 0, 0.0), m, FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _bwd(lib, _abi.Shape(0, 128, 2, 64, 0, 0.0), m, FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _bwd(lib, _abi.Shape(1, 128, 0, 64, 0, 0.0), m, FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _bwd(lib, _abi.Shape(1, 128, 2, 96, 0, 0.0), m, FAKE) == _abi.ERR_UNSUPPORTED
    assert _bwd(lib, _abi.Shape(1, 128, 2, 64, 3, 0.0), m, FAKE) == _abi.ERR_UNSUPPORTED
    assert _bwd(lib, _abi.Shape(1, 128, 2, 64, 0, float("nan")), m, FAKE) == \
        _abi.ERR_INVALID_ARGUMENT


def test_rejects_bad_masks(lib):
    s = _abi.Shape(1, 128, 2, 64, 0, 0.0)
    assert _bwd(lib, s, _abi.Mask(2, 16, 4), FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _bwd(lib, s, _abi.Mask(TF, 0, 4), FAKE) == _abi.ERR_INVALID_ARGUMENT
    assert _bwd(lib, s, _abi.Mask(BC, 16, 4), FAKE) == _abi.ERR_INVALID_ARGUMENT  # L = 64


@pytest.mark.parametrize("i", [0, 1, 2, 3, 4, 5, 7, 8, 9])
def test_rejects_null_and_misaligned_pointers(lib, i):
    s = _abi.Shape(1, 128, 2, 64, 0, 0.0)
    m = _abi.Mask(TF, 16, 4)
    ptrs = list(FAKE)
    ptrs[i] = None
    assert _bwd(lib, s, m, ptrs) == _abi.ERR_INVALID_ARGUMENT
    ptrs = list(FAKE)
    ptrs[i] += 8
    assert _bwd(lib, s, m, ptrs) == _abi.ERR_MISALIGNED


def test_misaligned_lse_cotangent_is_rejected(lib):
    # dlse may be null; when given it must be aligned like the rest
    s = _abi.Shape(1, 128, 2, 64, 0, 0.0)
    ptrs = list(FAKE)
    ptrs[6] += 4
    assert _bwd(lib, s, _abi.Mask(TF, 16, 4), ptrs) == _abi.ERR_MISALIGNED
    ptrs[0] = None  # and null dlse still leaves the other checks in force
    ptrs[6] = None
    assert _bwd(lib, s, _abi.Mask(TF, 16, 4), ptrs) == _abi.ERR_INVALID_ARGUMENT


@pytest.mark.parametrize("groups,L,n,code", [
    ([(8, 0, 8, 8, 8)], 8, 0, _abi.ERR_INVALID_ARGUMENT),
    ([(8, 0, 8, 8, 8)], 8, _abi.MAX_GROUPS + 1, _abi.ERR_UNSUPPORTED),
    ([(4, 0, 4, 4, 4), (7, 0, 8, 8, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),
    ([(8, 0, 5, 4, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),
    ([(8, 0, 4, 6, 9)], 8, None, _abi.ERR_INVALID_ARGUMENT),
    ([(4, 0, 4, 4, 4), (8, 2, 2, 5, 5)], 8, None, _abi.ERR_INVALID_ARGUMENT),
    (None, 8, 1, _abi.ERR_INVALID_ARGUMENT),
])
def test_groups_form_rejects_bad_tables(lib, groups, L, n, code):
    s = _abi.Shape(1, L, 2, 64, 0, 0.0)
    assert _bwd_groups(lib, s, groups, n, FAKE) == code
