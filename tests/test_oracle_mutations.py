"""Plant plausible mistakes in the oracle (on the CPU) and check that its pins
catch each one: the pins would fail for a dropped term, a wrong sign, an
off-by-one chunk index, a transposed operand or a missing scale."""
import math

import numpy as np
import pytest

import test_oracle_pins as pins
from oracle import attn_jvp_oracle as orc

TF = orc.TEACHER_FORCING


def _allowed_noisy_sees_own_clean_chunk(mode, c, n, i, j):
    # mistake: a noisy query in chunk i also sees clean chunk i
    base = orc.allowed.__wrapped__(mode, c, n, i, j)
    if mode != TF:
        return base
    i = np.asarray(i)
    j = np.asarray(j)
    nc = n * c
    extra = (i >= nc) & (j < nc) & ((j // c) == (i - nc) // c)
    return base | extra


def _allowed_block_causal_strict(mode, c, n, i, j):
    # mistake: block-causal without the own chunk on the diagonal
    if mode == orc.BLOCK_CAUSAL:
        return (np.asarray(j) // c) < (np.asarray(i) // c)
    return orc.allowed.__wrapped__(mode, c, n, i, j)


def _rows_variant(kind):
    def rows(q, k, v, tq, tk, tv, mode, c, n, scale, rows, block=64, groups=None):
        q, k, v, tq, tk, tv = (orc._as64(x) for x in (q, k, v, tq, tk, tv))
        L, d = q.shape
        s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
        rr = np.asarray(rows, dtype=np.int64)
        if groups is not None:
            M = orc.allowed_groups(groups, rr[:, None], np.arange(L)[None, :])
        else:
            M = orc.allowed(mode, c, n, rr[:, None], np.arange(L)[None, :])
        S = np.where(M, s * (q[rr] @ k.T), -np.inf)
        lse = np.logaddexp.reduce(S, axis=1)
        P = np.exp(S - lse[:, None])
        if kind == "tS_no_scale":
            tS = tq[rr] @ k.T + q[rr] @ tk.T
        elif kind == "tS_drop_qtk":
            tS = s * (tq[rr] @ k.T)
        else:
            tS = s * (tq[rr] @ k.T + q[rr] @ tk.T)
        tS = np.where(M, tS, 0.0)
        mu = (P * tS).sum(axis=1, keepdims=True)
        if kind == "mu_sign":
            tP = P * (tS + mu)
        else:
            tP = P * (tS - mu)
        O = P @ v
        if kind == "drop_p_tv":
            tO = tP @ v
        elif kind == "tv_transposed":
            tO = tP @ v + P @ tv[:, ::-1]
        else:
            tO = tP @ v + P @ tv
        return O, tO, lse
    return rows


PIN_CHECKS = [
    lambda: pins.test_mask_matches_hand_written("mask_tf_c2_n3.txt", TF, 2, 3),
    lambda: pins.test_mask_matches_hand_written("mask_bc_c2_n3.txt", orc.BLOCK_CAUSAL, 2, 3),
    lambda: pins.test_pair_count_closed_form(2, 3),
    lambda: pins.test_against_torch_autodiff(TF, 2, 3, 8, None),
    lambda: pins.test_against_torch_autodiff(orc.BLOCK_CAUSAL, 2, 3, 8, None),
    lambda: pins.test_finite_differences(TF),
    lambda: pins.test_zero_score_tangent_gives_p_tv(),
    lambda: pins.test_value_tangent_equal_to_value_gives_output(),
    lambda: pins.test_scaling_query_and_key_tangent(),
]
for case in pins._closed_form_cases():
    PIN_CHECKS.append(lambda case=case: pins.test_closed_form_cases(case))


def _caught(monkeypatch, attr, fn):
    monkeypatch.setattr(orc, attr, fn)
    failures = 0
    for check in PIN_CHECKS:
        try:
            check()
        except AssertionError:
            failures += 1
    return failures


@pytest.fixture(autouse=True)
def _wrap_allowed(monkeypatch):
    # keep a handle on the true predicate for the mutants that extend it
    true_allowed = orc.allowed
    if not hasattr(true_allowed, "__wrapped__"):
        def allowed(*a, **kw):
            return true_allowed(*a, **kw)
        allowed.__wrapped__ = true_allowed
        monkeypatch.setattr(orc, "allowed", allowed)
    yield


def test_unmutated_oracle_passes_every_pin():
    for check in PIN_CHECKS:
        check()


@pytest.mark.parametrize("mutant", [_allowed_noisy_sees_own_clean_chunk,
                                    _allowed_block_causal_strict])
def test_mask_mistakes_are_caught(monkeypatch, mutant):
    mutant.__wrapped__ = orc.allowed.__wrapped__
    assert _caught(monkeypatch, "allowed", mutant) > 0


@pytest.mark.parametrize("kind", ["tS_no_scale", "tS_drop_qtk", "mu_sign", "drop_p_tv",
                                  "tv_transposed"])
def test_jvp_mistakes_are_caught(monkeypatch, kind):
    assert _caught(monkeypatch, "attn_jvp_rows", _rows_variant(kind)) > 0


def test_correct_rewrite_is_not_flagged(monkeypatch):
    # the same formula written independently passes all pins (no false alarms)
    assert _caught(monkeypatch, "attn_jvp_rows", _rows_variant("none")) == 0


def _groups_row_boundary_off_by_one(groups, i, j):
    # mistake: the last row of each group is given the next group's keys
    i = np.asarray(i, dtype=np.int64)
    g = np.asarray(groups, dtype=np.int64).reshape(-1, 5)
    gi = np.minimum(np.searchsorted(g[:, 0], i + 1, side="right"), g.shape[0] - 1)
    j = np.asarray(j, dtype=np.int64)
    k0b, k0e, k1b, k1e = (g[gi, c] for c in range(1, 5))
    return ((j >= k0b) & (j < k0e)) | ((j >= k1b) & (j < k1e))


def _groups_end_inclusive(groups, i, j):
    # mistake: key ranges taken as closed intervals
    i = np.asarray(i, dtype=np.int64)
    g = np.asarray(groups, dtype=np.int64).reshape(-1, 5)
    gi = np.searchsorted(g[:, 0], i, side="right")
    j = np.asarray(j, dtype=np.int64)
    k0b, k0e, k1b, k1e = (g[gi, c] for c in range(1, 5))
    return ((j >= k0b) & (j <= k0e)) | ((j >= k1b) & (j <= k1e))


GROUP_PIN_CHECKS = [
    lambda: pins.test_group_mask_matches_hand_written(),
    lambda: pins.test_groups_against_torch_autodiff(),
]
for _m in (TF, orc.BLOCK_CAUSAL):
    for _c, _n in ((2, 3), (5, 4)):
        GROUP_PIN_CHECKS.append(
            lambda m=_m, c=_c, n=_n: pins.test_group_table_of_each_mode_gives_its_mask(m, c, n))


@pytest.mark.parametrize("mutant", [_groups_row_boundary_off_by_one, _groups_end_inclusive])
def test_group_mask_mistakes_are_caught(monkeypatch, mutant):
    monkeypatch.setattr(orc, "allowed_groups", mutant)
    failures = 0
    for check in GROUP_PIN_CHECKS:
        try:
            check()
        except (AssertionError, IndexError):
            failures += 1
    assert failures > 0


def test_group_pins_pass_unmutated():
    for check in GROUP_PIN_CHECKS:
        check()
