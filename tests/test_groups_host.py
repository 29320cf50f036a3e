"""Group-table masks on the host (no GPU): argument checks of
attn_jvp_fwd_groups (every call here fails validation, so nothing touches a
device) and the key-tile schedule the kernels run for a table.

The schedule is checked against the oracle's group predicate: every
admissible (row, key) pair of a query block lies in a listed key tile, every
tile flagged full is admissible for every row of the block, no tile is listed
twice, and for the teacher-forcing and block-causal tables the schedule is the
one the {mode, c, n} form gets.
"""
import ctypes

import numpy as np
import pytest

from attention_jvp_attn_b200 import _abi
from oracle import attn_jvp_oracle as orc

TF, BC = orc.TEACHER_FORCING, orc.BLOCK_CAUSAL


@pytest.fixture(scope="module")
def lib():
    from attention_jvp_attn_b200 import build
    build.build()
    return _abi.load()


FAKE = [0x10000 * (i + 1) for i in range(9)]  # never dereferenced: every call fails validation


def _call(lib, L, groups, n=None):
    shape = _abi.Shape(1, L, 2, 64, _abi.DTYPE_BF16, 0.0)
    arr = _abi.group_array(groups)
    return lib.attn_jvp_fwd_groups(ctypes.byref(shape), *FAKE[:6], arr,
                                   len(groups) if n is None else n, *FAKE[6:], None)


@pytest.mark.parametrize("groups,L,n,code", [
    ([(8, 0, 8, 8, 8)], 8, 0, _abi.ERR_INVALID_ARGUMENT),                     # no groups
    ([(8, 0, 8, 8, 8)], 8, _abi.MAX_GROUPS + 1, _abi.ERR_UNSUPPORTED),       # too many
    ([(4, 0, 4, 4, 4), (4, 0, 8, 8, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),  # rows not increasing
    ([(4, 0, 4, 4, 4), (7, 0, 8, 8, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),  # ends before L
    ([(4, 0, 4, 4, 4), (9, 0, 8, 8, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),  # ends after L
    ([(8, 3, 2, 8, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),                   # k0 reversed
    ([(8, 0, 5, 4, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),                   # ranges overlap
    ([(8, 0, 4, 6, 9)], 8, None, _abi.ERR_INVALID_ARGUMENT),                   # key past L
    ([(8, -1, 4, 6, 8)], 8, None, _abi.ERR_INVALID_ARGUMENT),                  # negative key
    ([(4, 0, 4, 4, 4), (8, 2, 2, 5, 5)], 8, None, _abi.ERR_INVALID_ARGUMENT),  # group without keys
])
def test_bad_tables_are_rejected(lib, groups, L, n, code):
    assert _call(lib, L, groups, n) == code


def test_null_table_is_rejected(lib):
    shape = _abi.Shape(1, 8, 2, 64, _abi.DTYPE_BF16, 0.0)
    assert lib.attn_jvp_fwd_groups(ctypes.byref(shape), *FAKE[:6], None, 1, *FAKE[6:], None) == \
        _abi.ERR_INVALID_ARGUMENT


def _sched(lib, groups, L, bm, bn, qt):
    arr = _abi.group_array(groups)
    cap = L // bn + 2
    tiles = (ctypes.c_int32 * cap)()
    full = (ctypes.c_uint8 * cap)()
    n = lib.attn_jvp_schedule_tiles_groups(arr, len(groups), L, bm, bn, qt, tiles, full, cap)
    assert 0 <= n <= cap
    return list(tiles[:n]), list(full[:n])


def _random_table(rng, L):
    cuts = sorted(set(rng.integers(1, L, size=rng.integers(0, 6)).tolist()) | {L})
    groups = []
    for end in cuts:
        pts = sorted(rng.integers(0, L + 1, size=4).tolist())
        a0, a1, b0, b1 = pts
        if rng.random() < 0.3:
            a0 = 0
        if a1 - a0 + b1 - b0 == 0:
            a0, a1 = 0, max(1, a1)
        groups.append((end, a0, a1, b0, b1))
    return groups


def _check_schedule(lib, groups, L, bm, bn):
    keys = np.arange(L)
    for qt in range((L + bm - 1) // bm):
        rows = np.arange(qt * bm, min(L, (qt + 1) * bm))
        M = orc.allowed_groups(groups, rows[:, None], keys[None, :])
        tiles, full = _sched(lib, groups, L, bm, bn, qt)
        assert len(set(tiles)) == len(tiles)
        needed = set(np.unique(np.nonzero(M)[1] // bn).tolist())
        assert needed <= set(tiles), (qt, needed - set(tiles))
        for kt, f in zip(tiles, full):
            if f:
                assert M[:, kt * bn:min(L, (kt + 1) * bn)].all()
                assert (kt + 1) * bn <= L


@pytest.mark.parametrize("seed", range(40))
def test_random_tables_schedule_covers_the_mask(lib, seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 700))
    groups = _random_table(rng, L)
    for bm, bn in ((128, 128), (256, 128), (32, 32)):
        _check_schedule(lib, groups, L, bm, bn)


@pytest.mark.parametrize("mode", [TF, BC])
@pytest.mark.parametrize("c,n", [(1, 3), (16, 4), (130, 3), (300, 2)])
def test_mode_tables_schedule_like_the_mode_form(lib, mode, c, n):
    groups = orc.group_table(mode, c, n)
    L = orc.seq_len(mode, c, n)
    mask = _abi.Mask(mode, c, n)
    for bm, bn in ((128, 128), (256, 128), (32, 32)):
        for qt in range((L + bm - 1) // bm):
            cap = L // bn + 2
            tiles = (ctypes.c_int32 * cap)()
            full = (ctypes.c_uint8 * cap)()
            nm = lib.attn_jvp_schedule_tiles(mask, L, bm, bn, qt, tiles, full, cap)
            assert (list(tiles[:nm]), list(full[:nm])) == _sched(lib, groups, L, bm, bn, qt)
        _check_schedule(lib, groups, L, bm, bn)
