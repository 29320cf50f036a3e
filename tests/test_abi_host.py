"""Host-side tests of the C ABI: the library loads without a GPU, exports every
symbol the header declares, rejects bad arguments before touching a device,
and its block-sparse mask schedule agrees with the oracle's explicit mask."""
import ctypes
import re

import numpy as np
import pytest

from attention_jvp_attn_b200 import _abi
import attention_jvp_attn_b200 as aj
from oracle import attn_jvp_oracle as orc

TF, BC = orc.TEACHER_FORCING, orc.BLOCK_CAUSAL


@pytest.fixture(scope="module")
def lib():
    from attention_jvp_attn_b200 import build
    build.build()
    return _abi.load()


def _declared_functions():
    src = open(_abi.HEADER_PATH).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(attn_jvp_[a-z0-9_]+)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_exports_every_declared_symbol(lib):
    names = _declared_functions()
    assert "attn_jvp_fwd" in names and "attn_jvp_schedule_tiles" in names
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.attn_jvp_version() >= 100
    for code in range(7):
        assert _abi.status_string(code)
    assert _abi.status_string(99) == "unknown status"


@pytest.mark.parametrize("mode,c,n", [(TF, 1, 1), (TF, 16, 4), (TF, 1560, 21), (TF, 4680, 7),
                                      (BC, 1560, 9), (BC, 3, 5), (TF, 256, 256)])
def test_unmasked_pairs_closed_form(lib, mode, c, n):
    got = aj.unmasked_pairs(mode, c, n)
    expect = c * c * n * (n + 1) // (1 if mode == TF else 2)
    assert got == expect
    if orc.seq_len(mode, c, n) <= 4096:
        assert got == orc.count_pairs_bruteforce(mode, c, n)


def test_unmasked_pairs_rejects_bad_mask(lib):
    assert aj.unmasked_pairs(7, 4, 4) == -1
    assert aj.unmasked_pairs(TF, 0, 4) == -1
    assert aj.unmasked_pairs(TF, 4, 0) == -1


def _check_schedule(mode, c, n, bm, bn):
    L = orc.seq_len(mode, c, n)
    M = orc.mask_matrix(mode, c, n)
    n_q = -(-L // bm)
    n_k = -(-L // bn)
    for qt in range(n_q):
        rows = M[qt * bm:min(L, (qt + 1) * bm)]
        tiles, full = aj.schedule_tiles(mode, c, n, L, bm, bn, qt)
        assert len(tiles) == len(set(tiles)), "a key tile listed twice"
        expect = []
        expect_full = {}
        for kt in range(n_k):
            blk = np.zeros((rows.shape[0], bn), dtype=bool)
            k1 = min(L, (kt + 1) * bn)
            blk[:, :k1 - kt * bn] = rows[:, kt * bn:k1]
            if blk.any():
                expect.append(kt)
                expect_full[kt] = bool(blk.all())
        assert sorted(tiles) == expect, (qt, tiles, expect)
        for kt, f in zip(tiles, full):
            assert bool(f) == expect_full[kt], (qt, kt)


@pytest.mark.parametrize("mode", [TF, BC])
@pytest.mark.parametrize("c,n", [(1, 1), (1, 7), (2, 3), (5, 4), (16, 4), (24, 5), (40, 3),
                                 (128, 2), (130, 3), (200, 2)])
@pytest.mark.parametrize("bm,bn", [(128, 128), (32, 32), (16, 64), (64, 16)])
def test_schedule_matches_explicit_mask(lib, mode, c, n, bm, bn):
    _check_schedule(mode, c, n, bm, bn)


def test_schedule_of_framewise_workload_spot_checks(lib):
    # 21 frames x 1560 tokens, packed clean|noisy: sample query tiles across
    # chunk boundaries and the ragged tail against the explicit mask rows.
    mode, c, n, bm, bn = TF, 1560, 21, 128, 128
    L = orc.seq_len(mode, c, n)
    keys = np.arange(L)
    for qt in (0, 12, 13, 255, 256, 257, 300, 511):
        rows = np.arange(qt * bm, min(L, (qt + 1) * bm))
        Mr = orc.allowed(mode, c, n, rows[:, None], keys[None, :])
        tiles, full = aj.schedule_tiles(mode, c, n, L, bm, bn, qt)
        n_k = -(-L // bn)
        expect = [kt for kt in range(n_k) if Mr[:, kt * bn:(kt + 1) * bn].any()]
        assert sorted(tiles) == expect
        for kt, f in zip(tiles, full):
            blk = Mr[:, kt * bn:(kt + 1) * bn]
            assert bool(f) == (blk.shape[1] == bn and bool(blk.all()))


def test_schedule_rejects_bad_arguments(lib):
    assert lib.attn_jvp_schedule_tiles(_abi.Mask(TF, 4, 2), 16, 8, 8, 2, None, None, 0) == -1  # qtile out of range
    assert lib.attn_jvp_schedule_tiles(_abi.Mask(TF, 4, 2), 15, 8, 8, 0, None, None, 0) == -1  # L mismatch
    assert lib.attn_jvp_schedule_tiles(_abi.Mask(TF, 4, 2), 16, 0, 8, 0, None, None, 0) == -1
    assert lib.attn_jvp_schedule_tiles(_abi.Mask(TF, 4, 2), 16, 8, 8, 0, None, None, 4) == -1  # null arrays


# ---- argument validation (returns before any device is touched) -----------

def _call(lib, shape, mask, ptrs):
    return lib.attn_jvp_fwd(ctypes.byref(shape) if shape is not None else None, *ptrs[:6], mask,
                            *ptrs[6:9], None)


GOOD = [0x10000 * (i + 1) for i in range(9)]  # never dereferenced: each case fails validation


def test_rejects_bad_shapes(lib):
    m = _abi.Mask(TF, 16, 4)
    assert _call(lib, None, m, GOOD) == _abi.ERR_INVALID_ARGUMENT
    assert _call(lib, _abi.Shape(1, 127, 2, 64, 0, 0.0), m, GOOD) == _abi.ERR_INVALID_ARGUMENT
    assert _call(lib, _abi.Shape(0, 128, 2, 64, 0, 0.0), m, GOOD) == _abi.ERR_INVALID_ARGUMENT
    assert _call(lib, _abi.Shape(1, 128, 0, 64, 0, 0.0), m, GOOD) == _abi.ERR_INVALID_ARGUMENT
    assert _call(lib, _abi.Shape(1, 128, 2, 96, 0, 0.0), m, GOOD) == _abi.ERR_UNSUPPORTED
    assert _call(lib, _abi.Shape(1, 128, 2, 64, 3, 0.0), m, GOOD) == _abi.ERR_UNSUPPORTED
    assert _call(lib, _abi.Shape(1, 128, 2, 64, 0, float("inf")), m, GOOD) == _abi.ERR_INVALID_ARGUMENT


def test_rejects_bad_masks(lib):
    s = _abi.Shape(1, 128, 2, 64, 0, 0.0)
    assert _call(lib, s, _abi.Mask(2, 16, 4), GOOD) == _abi.ERR_INVALID_ARGUMENT
    assert _call(lib, s, _abi.Mask(TF, 0, 4), GOOD) == _abi.ERR_INVALID_ARGUMENT
    assert _call(lib, s, _abi.Mask(TF, 16, -1), GOOD) == _abi.ERR_INVALID_ARGUMENT
    assert _call(lib, s, _abi.Mask(BC, 16, 4), GOOD) == _abi.ERR_INVALID_ARGUMENT  # L = 64 expected


def test_rejects_null_and_misaligned_pointers(lib):
    s = _abi.Shape(1, 128, 2, 64, 0, 0.0)
    m = _abi.Mask(TF, 16, 4)
    for i in range(9):
        ptrs = list(GOOD)
        ptrs[i] = None
        assert _call(lib, s, m, ptrs) == _abi.ERR_INVALID_ARGUMENT
        ptrs = list(GOOD)
        ptrs[i] += 8
        assert _call(lib, s, m, ptrs) == _abi.ERR_MISALIGNED


def _round256(x):
    return (x + 255) // 256 * 256


def test_staging_bytes(lib):
    # heads go in up to 16 chunks through two staging slots, each holding the
    # 8 tensors and the LSE of one chunk (256-byte aligned pieces)
    s = _abi.Shape(2, 128, 3, 64, 0, 0.0)  # 3 chunks of 1 head
    slot = 8 * _round256(2 * 128 * 1 * 64 * 2) + _round256(2 * 1 * 128 * 4)
    assert lib.attn_jvp_host_staging_bytes(ctypes.byref(s)) == 2 * slot
    s = _abi.Shape(1, 100, 12, 128, 1, 0.0)  # fp32, 12 chunks of 1 head
    slot = 8 * _round256(100 * 1 * 128 * 4) + _round256(1 * 100 * 4)
    assert lib.attn_jvp_host_staging_bytes(ctypes.byref(s)) == 2 * slot
    s = _abi.Shape(1, 100, 40, 64, 0, 0.0)  # 14 chunks of 3 heads (the last one of 1)
    slot = 8 * _round256(100 * 3 * 64 * 2) + _round256(3 * 100 * 4)
    assert lib.attn_jvp_host_staging_bytes(ctypes.byref(s)) == 2 * slot
    s = _abi.Shape(1, 100, 1, 64, 0, 0.0)  # one head: one slot of the whole problem
    assert lib.attn_jvp_host_staging_bytes(ctypes.byref(s)) == \
        8 * _round256(100 * 64 * 2) + _round256(100 * 4)
    assert lib.attn_jvp_host_staging_bytes(ctypes.byref(_abi.Shape(0, 1, 1, 64, 0, 0.0))) == 0


def test_debug_wait_settings_are_checked(lib):
    # test-only bounded-wait settings: checked on the host, restored at the end
    assert lib.attn_jvp_debug_wait(-1, -1) == _abi.ERR_INVALID_ARGUMENT
    assert lib.attn_jvp_debug_wait(0, -2) == _abi.ERR_INVALID_ARGUMENT
    assert lib.attn_jvp_debug_wait(61 * 10**9, -1) == _abi.ERR_INVALID_ARGUMENT
    assert lib.attn_jvp_debug_wait(2_000_000, 3) == _abi.OK
    assert lib.attn_jvp_debug_wait(0, -1) == _abi.OK


@pytest.mark.parametrize("mode", [TF, BC])
@pytest.mark.parametrize("c,n", [(1, 1), (1, 7), (5, 4), (24, 5), (100, 3), (128, 2), (130, 3),
                                 (150, 3), (200, 2), (1560, 2)])
@pytest.mark.parametrize("bm,bn", [(128, 128), (64, 128), (32, 32)])
def test_key_tile_query_bounds_cover_the_explicit_mask(lib, mode, c, n, bm, bn):
    """The backward's dK/dV kernel scans only the query tiles in these bounds
    for a key tile: every query tile with an admissible pair in the key tile
    (from the oracle's explicit mask) must lie inside them, and for these
    closed-form masks the lower bound is the first such tile."""
    L = orc.seq_len(mode, c, n)
    M = orc.mask_matrix(mode, c, n)
    n_q = -(-L // bm)
    for kt in range(-(-L // bn)):
        lo, hi = aj.key_tile_query_bounds(mode, c, n, L, bm, bn, kt)
        cols = M[:, kt * bn:min(L, (kt + 1) * bn)]
        seen = [qt for qt in range(n_q) if cols[qt * bm:min(L, (qt + 1) * bm)].any()]
        assert 0 <= lo <= hi < n_q, (kt, lo, hi)
        if seen:
            assert lo == seen[0] and seen[-1] <= hi, (kt, lo, hi, seen[0], seen[-1])


def test_key_tile_query_bounds_rejects_bad_arguments(lib):
    with pytest.raises(ValueError):
        aj.key_tile_query_bounds(TF, 16, 2, 64, 128, 128, 1)  # key tile past L
    with pytest.raises(ValueError):
        aj.key_tile_query_bounds(TF, 16, 2, 65, 128, 128, 0)  # L does not match the mask
    with pytest.raises(ValueError):
        aj.key_tile_query_bounds(TF, 16, 2, 64, 0, 128, 0)
