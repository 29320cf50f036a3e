"""Pins for the float64 oracle, against facts that do not come from it.

* hand-written masks (tests/golden/mask_*.txt) and pair-count closed forms
  pin the mask predicate;
* hand-derived outputs (tests/golden/closed_form.json) pin O, LSE and tO;
* forward-mode autodiff through torch's float64 softmax attention (a library
  routine) pins the whole JVP on random inputs;
* central finite differences of the oracle's primal output pin tO;
* invariants: tq=tk=0 gives tO = P tv, q=0 gives uniform P, linearity in the
  tangent, shift invariance of softmax, tangent (0,0,v) gives tO = O,
  tangent (q,k,0) doubles tS, and mask identities (clean half = block-causal
  on the clean half; noisy chunk = dense attention over its visible keys).

Each pin is chosen so that a plausible slip in the oracle (a dropped term,
a wrong sign, an off-by-one chunk index, a transposed operand) fails it.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.func import jvp
from torch.nn.attention import SDPBackend, sdpa_kernel

from oracle import attn_jvp_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TF, BC = orc.TEACHER_FORCING, orc.BLOCK_CAUSAL


def _read_mask(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([ch == "1" for ch in line])
    return np.array(rows, dtype=bool)


@pytest.mark.parametrize("fname,mode,c,n", [
    ("mask_tf_c2_n3.txt", TF, 2, 3),
    ("mask_bc_c2_n3.txt", BC, 2, 3),
    ("mask_tf_c1_n2.txt", TF, 1, 2),
    ("mask_tf_c3_n1.txt", TF, 3, 1),
])
def test_mask_matches_hand_written(fname, mode, c, n):
    assert np.array_equal(orc.mask_matrix(mode, c, n), _read_mask(fname))


GROUPS_EXAMPLE = [(2, 0, 3, 6, 8), (5, 1, 2, 4, 6), (8, 5, 8, 8, 8)]


def test_group_mask_matches_hand_written():
    assert np.array_equal(orc.mask_matrix_groups(GROUPS_EXAMPLE),
                          _read_mask("mask_groups_example.txt"))


@pytest.mark.parametrize("mode", [TF, BC])
@pytest.mark.parametrize("c,n", [(1, 1), (2, 3), (3, 1), (5, 4)])
def test_group_table_of_each_mode_gives_its_mask(mode, c, n):
    # two restatements of the same mask (chunk rule vs. per-group key ranges)
    assert np.array_equal(orc.mask_matrix_groups(orc.group_table(mode, c, n)),
                          orc.mask_matrix(mode, c, n))


def test_groups_path_matches_mode_path_numerically():
    rng = np.random.default_rng(5)
    c, n, d = 3, 3, 8
    L = 2 * n * c
    x = [rng.standard_normal((1, L, 2, d)) for _ in range(6)]
    a = orc.attn_jvp_dense(*x, TF, c, n)
    b = orc.attn_jvp_dense(*x, TF, c, n, groups=orc.group_table(TF, c, n))
    for u, w in zip(a, b):
        assert np.array_equal(u, w)


def test_groups_against_torch_autodiff():
    # JVP of the library's softmax attention (MATH backend) under the
    # hand-written group mask
    import torch
    from torch.func import jvp
    rng = np.random.default_rng(11)
    M = _read_mask("mask_groups_example.txt")
    L, d = M.shape[0], 4
    q, k, v, tq, tk, tv = (rng.standard_normal((L, d)) for _ in range(6))
    O, tO, lse = orc.attn_jvp_rows(q, k, v, tq, tk, tv, TF, 1, 1, None, np.arange(L),
                                   groups=GROUPS_EXAMPLE)
    mask = torch.from_numpy(M)

    def f(qq, kk, vv):
        with torch.nn.attention.sdpa_kernel(torch.nn.attention.SDPBackend.MATH):
            return torch.nn.functional.scaled_dot_product_attention(
                qq[None, None], kk[None, None], vv[None, None], attn_mask=mask)[0, 0]

    T = lambda a: torch.from_numpy(a)
    o_ref, to_ref = jvp(f, (T(q), T(k), T(v)), (T(tq), T(tk), T(tv)))
    assert np.allclose(O, o_ref.numpy(), atol=1e-12, rtol=1e-10)
    assert np.allclose(tO, to_ref.numpy(), atol=1e-12, rtol=1e-10)
    s = 1.0 / math.sqrt(d)
    S = np.where(M, s * q @ k.T, -np.inf)
    assert np.allclose(lse, np.log(np.exp(S).sum(axis=1)), atol=1e-12)


@pytest.mark.parametrize("c", [1, 2, 3, 5, 16])
@pytest.mark.parametrize("n", [1, 2, 3, 7])
def test_pair_count_closed_form(c, n):
    # clean half: c^2 n(n+1)/2 pairs; noisy half: c^2 n(n-1)/2 (clean keys of
    # earlier chunks) + c^2 n (own chunk); total c^2 n(n+1).
    assert orc.count_pairs_bruteforce(TF, c, n) == c * c * n * (n + 1)
    assert orc.count_pairs_bruteforce(BC, c, n) == c * c * n * (n + 1) // 2


def test_every_row_sees_its_own_chunk():
    for mode in (TF, BC):
        for c, n in ((1, 1), (3, 4), (16, 4)):
            M = orc.mask_matrix(mode, c, n)
            L = M.shape[0]
            assert M[np.arange(L), np.arange(L)].all()


def _val(x):
    if isinstance(x, str):
        return float(eval(x, {"__builtins__": {}}, {"ln2": math.log(2), "ln3": math.log(3),
                                                  "ln4": math.log(4)}))
    return float(x)


def _arr(a):
    return np.array([[_val(x) for x in row] for row in a]) if isinstance(a[0], list) \
        else np.array([_val(x) for x in a])


def _closed_form_cases():
    with open(os.path.join(GOLDEN, "closed_form.json")) as f:
        return json.load(f)["cases"]


@pytest.mark.parametrize("case", _closed_form_cases(), ids=lambda c: c["name"])
def test_closed_form_cases(case):
    t = {k: _arr(case[k]) for k in ("q", "k", "v", "tq", "tk", "tv")}
    L = t["q"].shape[0]
    O, tO, lse = orc.attn_jvp_rows(t["q"], t["k"], t["v"], t["tq"], t["tk"], t["tv"],
                                   case["mode"], case["chunk_tokens"], case["n_chunks"],
                                   case["scale"], range(L))
    np.testing.assert_allclose(O, _arr(case["O"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, _arr(case["LSE"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(tO, _arr(case["tO"]), rtol=0, atol=1e-12)


def _rand(shape, seed):
    g = np.random.default_rng(seed)
    return [g.standard_normal(shape) for _ in range(6)]


def _torch_reference(q, k, v, tq, tk, tv, mask, scale):
    """Forward-mode autodiff through torch's math-backend softmax attention."""
    def f(a, b, c):
        return F.scaled_dot_product_attention(a, b, c, attn_mask=mask, scale=scale)
    to_t = lambda x: torch.from_numpy(x).permute(1, 0, 2).unsqueeze(0)  # [1,H,L,d]
    with sdpa_kernel(SDPBackend.MATH):
        o, to = jvp(f, (to_t(q), to_t(k), to_t(v)), (to_t(tq), to_t(tk), to_t(tv)))
    back = lambda x: x.squeeze(0).permute(1, 0, 2).numpy()
    return back(o), back(to)


@pytest.mark.parametrize("mode,c,n,d,scale", [
    (TF, 2, 3, 8, None), (TF, 3, 4, 5, 0.37), (BC, 2, 3, 8, None), (BC, 4, 5, 16, 1.3),
    (TF, 5, 1, 4, None), (BC, 7, 1, 4, None),
])
def test_against_torch_autodiff(mode, c, n, d, scale):
    L = orc.seq_len(mode, c, n)
    H = 2
    q, k, v, tq, tk, tv = _rand((L, H, d), seed=L * 31 + d)
    mask = torch.from_numpy(orc.mask_matrix(mode, c, n))
    s = 1.0 / math.sqrt(d) if scale is None else scale
    o_ref, to_ref = _torch_reference(q, k, v, tq, tk, tv, mask, s)
    O, tO, lse = orc.attn_jvp_dense(q[None], k[None], v[None], tq[None], tk[None], tv[None],
                                    mode, c, n, scale)
    np.testing.assert_allclose(O[0], o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(tO[0], to_ref, rtol=1e-11, atol=1e-11)
    # LSE against a direct logsumexp over the hand-written-pinned mask
    S = s * np.einsum("ihd,jhd->hij", q, k)
    S = np.where(mask.numpy()[None], S, -np.inf)
    np.testing.assert_allclose(lse[0], np.logaddexp.reduce(S, axis=2), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("mode", [TF, BC])
def test_finite_differences(mode):
    c, n, d = 2, 3, 8
    L = orc.seq_len(mode, c, n)
    q, k, v, tq, tk, tv = (x[None] for x in _rand((L, 1, d), seed=5 + mode))
    eps = 1e-6
    Op, _ = orc.attn_forward_dense(q + eps * tq, k + eps * tk, v + eps * tv, mode, c, n)
    Om, _ = orc.attn_forward_dense(q - eps * tq, k - eps * tk, v - eps * tv, mode, c, n)
    fd = (Op - Om) / (2 * eps)
    _, tO, _ = orc.attn_jvp_dense(q, k, v, tq, tk, tv, mode, c, n)
    np.testing.assert_allclose(tO, fd, rtol=0, atol=1e-8)


def _setup(mode=TF, c=3, n=4, d=6, H=2, seed=11):
    L = orc.seq_len(mode, c, n)
    return [x[None] for x in _rand((L, H, d), seed)], (mode, c, n)


def test_zero_score_tangent_gives_p_tv():
    (q, k, v, tq, tk, tv), m = _setup()
    z = np.zeros_like(q)
    _, tO, _ = orc.attn_jvp_dense(q, k, v, z, z, tv, *m)
    O_tv, _ = orc.attn_forward_dense(q, k, tv, *m)      # P @ tv
    np.testing.assert_allclose(tO, O_tv, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("mode", [TF, BC])
def test_zero_query_gives_uniform_attention(mode):
    (q, k, v, tq, tk, tv), m = _setup(mode=mode)
    z = np.zeros_like(q)
    O, _, lse = orc.attn_jvp_dense(z, k, v, tq, tk, tv, *m)
    M = orc.mask_matrix(*m)
    cnt = M.sum(axis=1)
    for h in range(q.shape[2]):
        mean_v = (M.astype(float) @ v[0, :, h]) / cnt[:, None]
        np.testing.assert_allclose(O[0, :, h], mean_v, rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(lse[0, h], np.log(cnt), rtol=1e-13, atol=1e-13)


def test_linearity_in_tangent():
    (q, k, v, tq, tk, tv), m = _setup()
    (_, _, _, uq, uk, uv), _ = _setup(seed=99)
    a, b = 0.7, -1.9
    _, t1, _ = orc.attn_jvp_dense(q, k, v, tq, tk, tv, *m)
    _, t2, _ = orc.attn_jvp_dense(q, k, v, uq, uk, uv, *m)
    _, t3, _ = orc.attn_jvp_dense(q, k, v, a * tq + b * uq, a * tk + b * uk, a * tv + b * uv, *m)
    np.testing.assert_allclose(t3, a * t1 + b * t2, rtol=1e-11, atol=1e-11)


def test_value_tangent_equal_to_value_gives_output():
    (q, k, v, tq, tk, tv), m = _setup()
    z = np.zeros_like(q)
    O, tO, _ = orc.attn_jvp_dense(q, k, v, z, z, v, *m)
    np.testing.assert_allclose(tO, O, rtol=1e-13, atol=1e-13)


def test_scaling_query_and_key_tangent():
    # tangent (q, k, 0): tS = 2 S, so tO equals twice the tO of tangent (q, 0, 0),
    # and tangent (q,0,0) equals tangent (0,k,0) since both give tS = S.
    (q, k, v, tq, tk, tv), m = _setup()
    z = np.zeros_like(q)
    _, t_qk, _ = orc.attn_jvp_dense(q, k, v, q, k, z, *m)
    _, t_q, _ = orc.attn_jvp_dense(q, k, v, q, z, z, *m)
    _, t_k, _ = orc.attn_jvp_dense(q, k, v, z, k, z, *m)
    np.testing.assert_allclose(t_qk, 2 * t_q, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(t_q, t_k, rtol=1e-12, atol=1e-12)
    # tangent (q,0,0) is d/de of O(q(1+e)): compare with a finite difference
    eps = 1e-6
    Op, _ = orc.attn_forward_dense(q * (1 + eps), k, v, *m)
    Om, _ = orc.attn_forward_dense(q * (1 - eps), k, v, *m)
    np.testing.assert_allclose(t_q, (Op - Om) / (2 * eps), rtol=0, atol=1e-8)


def test_softmax_shift_invariance():
    # tk rows all equal to one vector u and tq = 0: tS is constant along keys,
    # so tP = 0 and tO = P tv.
    (q, k, v, tq, tk, tv), m = _setup()
    u = np.random.default_rng(3).standard_normal(q.shape[-1])
    tk_const = np.broadcast_to(u, q.shape).copy()
    z = np.zeros_like(q)
    _, tO, _ = orc.attn_jvp_dense(q, k, v, z, tk_const, tv, *m)
    O_tv, _ = orc.attn_forward_dense(q, k, tv, *m)
    np.testing.assert_allclose(tO, O_tv, rtol=1e-12, atol=1e-12)


def test_clean_half_equals_block_causal():
    c, n = 3, 4
    (q, k, v, tq, tk, tv), _ = _setup(mode=TF, c=c, n=n)
    nc = n * c
    O, tO, lse = orc.attn_jvp_dense(q, k, v, tq, tk, tv, TF, c, n)
    sub = [x[:, :nc] for x in (q, k, v, tq, tk, tv)]
    O2, tO2, lse2 = orc.attn_jvp_dense(*sub, BC, c, n)
    np.testing.assert_allclose(O[:, :nc], O2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(tO[:, :nc], tO2, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(lse[:, :, :nc], lse2, rtol=1e-13, atol=1e-13)


def test_noisy_chunk_equals_dense_attention_over_visible_keys():
    c, n = 3, 4
    (q, k, v, tq, tk, tv), _ = _setup(mode=TF, c=c, n=n)
    nc = n * c
    O, tO, lse = orc.attn_jvp_dense(q, k, v, tq, tk, tv, TF, c, n)
    d = q.shape[3]
    for i in range(n):
        qs = slice(nc + i * c, nc + (i + 1) * c)
        keys = np.r_[np.arange(0, i * c), np.arange(nc + i * c, nc + (i + 1) * c)]
        Lk = len(keys)
        for h in range(q.shape[2]):
            # one chunk of Lk tokens in block-causal mode = dense attention;
            # the noisy queries sit in the first c query slots
            qp = np.zeros((Lk, d)); qp[:c] = q[0, qs, h]
            tqp = np.zeros((Lk, d)); tqp[:c] = tq[0, qs, h]
            Od, tOd, lsed = orc.attn_jvp_rows(qp, k[0, keys, h], v[0, keys, h], tqp,
                                              tk[0, keys, h], tv[0, keys, h],
                                              BC, Lk, 1, None, range(c))
            np.testing.assert_allclose(O[0, qs, h], Od, rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(tO[0, qs, h], tOd, rtol=1e-13, atol=1e-13)
            np.testing.assert_allclose(lse[0, h, qs], lsed, rtol=1e-13, atol=1e-13)


def test_single_chunk_block_causal_is_dense_softmax_attention():
    # n=1 block-causal is plain dense attention: compare with torch SDPA (no mask)
    L, H, d = 9, 2, 4
    q, k, v, tq, tk, tv = _rand((L, H, d), seed=21)
    o_ref, to_ref = _torch_reference(q, k, v, tq, tk, tv, None, 0.5)
    O, tO, _ = orc.attn_jvp_dense(q[None], k[None], v[None], tq[None], tk[None], tv[None],
                                  BC, L, 1, 0.5)
    np.testing.assert_allclose(O[0], o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(tO[0], to_ref, rtol=1e-11, atol=1e-11)


def test_rows_subset_matches_dense():
    (q, k, v, tq, tk, tv), m = _setup(c=5, n=3)
    O, tO, lse = orc.attn_jvp_dense(q, k, v, tq, tk, tv, *m)
    rows = [0, 4, 5, 14, 15, 29]
    o_, to_, l_ = orc.attn_jvp_rows(q[0, :, 1], k[0, :, 1], v[0, :, 1], tq[0, :, 1],
                                    tk[0, :, 1], tv[0, :, 1], *m, None, rows, block=4)
    np.testing.assert_array_equal(o_, O[0, rows, 1])
    np.testing.assert_array_equal(to_, tO[0, rows, 1])
    np.testing.assert_array_equal(l_, lse[0, 1, rows])


def test_bf16_inputs_promote_bit_exactly():
    x = torch.randn(3, 4, 2, 8).to(torch.bfloat16)
    y = orc._as64(x)
    assert y.dtype == np.float64
    assert np.array_equal(y, x.float().numpy().astype(np.float64))
