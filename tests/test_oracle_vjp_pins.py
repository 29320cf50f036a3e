"""Pins of the oracle's backward (vector-Jacobian product) of the masked
attention, against values that do not come from the oracle's backward itself:

- reverse-mode autodiff of torch's math-backend softmax attention under the
  same mask (dQ, dK, dV), and of a masked logsumexp (the dLSE term);
- the adjoint identity with the oracle's forward JVP, which is pinned on its
  own: <dO, J t> = <J^T dO, t> for every tangent t;
- central finite differences of a scalar loss of the forward output;
- special cases with closed forms (one admissible key per row; zero output
  cotangent; a dLSE cotangent on a query of zeros).

The mutation tests at the end plant mistakes in a copy of the backward (a
dropped Delta term, a transposed dS, a missing scale, a wrong dLSE sign) and
check that these pins catch each.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.nn.attention import SDPBackend, sdpa_kernel

from oracle import attn_jvp_oracle as orc

TF, BC = orc.TEACHER_FORCING, orc.BLOCK_CAUSAL
GROUPS = [(3, 0, 3, 3, 3), (7, 1, 2, 4, 9), (9, 0, 0, 5, 9)]


def _rand(L, H, d, seed, n=4):
    g = np.random.default_rng(seed)
    return [g.standard_normal((1, L, H, d)) for _ in range(n)]


def _mask(mode, c, n, groups):
    return orc.mask_matrix_groups(groups) if groups is not None else orc.mask_matrix(mode, c, n)


CASES = [  # mode, c, n, d, H, scale, groups
    (TF, 2, 3, 8, 2, None, None),
    (TF, 3, 2, 5, 1, 0.41, None),
    (BC, 2, 4, 8, 2, None, None),
    (BC, 5, 1, 4, 1, 1.3, None),
    (TF, 1, 1, 4, 2, None, GROUPS),
]


def _ids(c):
    return f"{'groups' if c[6] else ('tf' if c[0] == TF else 'bc')}_c{c[1]}_n{c[2]}_d{c[3]}"


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_against_torch_reverse_autodiff(case):
    mode, c, n, d, H, scale, groups = case
    M = _mask(mode, c, n, groups)
    L = M.shape[0]
    q, k, v, do = _rand(L, H, d, seed=L * 7 + d)
    dQ, dK, dV = orc.attn_vjp_dense(q, k, v, do, mode, c, n, scale, groups=groups)
    s = 1.0 / math.sqrt(d) if scale is None else scale
    T = lambda x: torch.from_numpy(x[0]).permute(1, 0, 2).unsqueeze(0).requires_grad_(True)
    tq, tk, tv = T(q), T(k), T(v)
    with sdpa_kernel(SDPBackend.MATH):
        o = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(M), scale=s)
    o.backward(torch.from_numpy(do[0]).permute(1, 0, 2).unsqueeze(0))
    back = lambda t: t.grad.squeeze(0).permute(1, 0, 2).numpy()[None]
    np.testing.assert_allclose(dQ, back(tq), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, back(tk), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, back(tv), rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_lse_cotangent_against_autodiff(case):
    # only dLSE (dO = 0): autodiff of torch.logsumexp over the masked scores
    mode, c, n, d, H, scale, groups = case
    M = _mask(mode, c, n, groups)
    L = M.shape[0]
    q, k, v, _ = _rand(L, H, d, seed=L * 3 + d)
    dlse = np.random.default_rng(L).standard_normal((1, H, L))
    zero = np.zeros_like(q)
    dQ, dK, dV = orc.attn_vjp_dense(q, k, v, zero, mode, c, n, scale, dlse=dlse, groups=groups)
    s = 1.0 / math.sqrt(d) if scale is None else scale
    for h in range(H):
        tq = torch.from_numpy(q[0, :, h]).requires_grad_(True)
        tk = torch.from_numpy(k[0, :, h]).requires_grad_(True)
        S = (s * tq @ tk.T).masked_fill(~torch.from_numpy(M), float("-inf"))
        torch.logsumexp(S, dim=1).backward(torch.from_numpy(dlse[0, h]))
        np.testing.assert_allclose(dQ[0, :, h], tq.grad.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(dK[0, :, h], tk.grad.numpy(), rtol=1e-10, atol=1e-12)
    assert not dV.any()


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_adjoint_of_the_pinned_jvp(case):
    # <dO, tO(t)> = <dQ, tq> + <dK, tk> + <dV, tv> for random tangents t
    mode, c, n, d, H, scale, groups = case
    M = _mask(mode, c, n, groups)
    L = M.shape[0]
    q, k, v, do, tq, tk, tv = _rand(L, H, d, seed=L * 11 + d, n=7)
    _, tO, _ = orc.attn_jvp_dense(q, k, v, tq, tk, tv, mode, c, n, scale, groups=groups)
    dQ, dK, dV = orc.attn_vjp_dense(q, k, v, do, mode, c, n, scale, groups=groups)
    lhs = float((do * tO).sum())
    rhs = float((dQ * tq).sum() + (dK * tk).sum() + (dV * tv).sum())
    assert abs(lhs - rhs) <= 1e-11 * (1.0 + abs(lhs))
    # the same identity through each input alone
    z = np.zeros_like(q)
    for tang, grad in (((tq, z, z), dQ), ((z, tk, z), dK), ((z, z, tv), dV)):
        _, t1, _ = orc.attn_jvp_dense(q, k, v, *tang, mode, c, n, scale, groups=groups)
        g = next(t for t in tang if t is not z)
        assert abs(float((do * t1).sum()) - float((grad * g).sum())) <= 1e-11 * (1 + abs(lhs))


@pytest.mark.parametrize("mode", [TF, BC])
def test_finite_differences_of_a_scalar_loss(mode):
    # loss = <W, O> + <w, LSE>; its gradient is the VJP with dO = W, dLSE = w
    c, n, d = 2, 3, 6
    L = orc.seq_len(mode, c, n)
    q, k, v, W = _rand(L, 1, d, seed=40 + mode)
    w = np.random.default_rng(9).standard_normal((1, 1, L))
    dQ, dK, dV = orc.attn_vjp_dense(q, k, v, W, mode, c, n, dlse=w)

    def loss(qq, kk, vv):
        O, lse = orc.attn_forward_dense(qq, kk, vv, mode, c, n)
        return float((W * O).sum() + (w * lse).sum())

    eps = 1e-6
    rng = np.random.default_rng(3)
    for _ in range(6):
        which = int(rng.integers(3))
        idx = (0, int(rng.integers(L)), 0, int(rng.integers(d)))
        args = [q.copy(), k.copy(), v.copy()]
        args[which][idx] += eps
        fp = loss(*args)
        args[which][idx] -= 2 * eps
        fm = loss(*args)
        fd = (fp - fm) / (2 * eps)
        assert abs(fd - (dQ, dK, dV)[which][idx]) <= 1e-7, (which, idx)


def test_one_admissible_key_per_row():
    # groups that admit only key j = i: P = I, so dV = dO and dQ = dK = 0
    L, d = 6, 4
    groups = [(i + 1, i, i + 1, i + 1, i + 1) for i in range(L)]
    q, k, v, do = _rand(L, 2, d, seed=5)
    dQ, dK, dV = orc.attn_vjp_dense(q, k, v, do, TF, 1, 1, groups=groups)
    np.testing.assert_array_equal(dV, do)
    assert not dQ.any() and not dK.any()


def test_zero_cotangent_gives_zero_gradients():
    q, k, v, _ = _rand(12, 2, 4, seed=6)
    g = orc.attn_vjp_dense(q, k, v, np.zeros_like(q), TF, 2, 3)
    assert all(not x.any() for x in g)


def test_lse_cotangent_on_a_zero_query():
    # q = 0 gives uniform P over the admissible keys; with dO = 0 and dLSE = 1,
    # dQ_i = s * mean of the admissible k_j, and dK = 0 (it is s dS^T q)
    c, n, d = 2, 3, 4
    L = orc.seq_len(BC, c, n)
    _, k, v, _ = _rand(L, 1, d, seed=8)
    z = np.zeros_like(k)
    dQ, dK, dV = orc.attn_vjp_dense(z, k, v, z, BC, c, n, dlse=np.ones((1, 1, L)))
    M = orc.mask_matrix(BC, c, n).astype(float)
    mean_k = (M @ k[0, :, 0]) / M.sum(axis=1)[:, None]
    np.testing.assert_allclose(dQ[0, :, 0], mean_k / math.sqrt(d), rtol=1e-13, atol=1e-14)
    assert not dK.any() and not dV.any()


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_sampled_rows_and_columns_match_the_dense_backward(case):
    # the row- and column-sampled forms used on large workloads give the same
    # numbers as the pinned dense backward
    mode, c, n, d, H, scale, groups = case
    M = _mask(mode, c, n, groups)
    L = M.shape[0]
    q, k, v, do = _rand(L, H, d, seed=L * 5 + d)
    dlse = np.random.default_rng(L + 1).standard_normal((1, H, L))
    dQ, dK, dV = orc.attn_vjp_dense(q, k, v, do, mode, c, n, scale, dlse=dlse, groups=groups)
    rng = np.random.default_rng(2)
    rows = np.unique(np.concatenate([[0, L - 1], rng.integers(0, L, 5)]))
    cols = np.unique(np.concatenate([[0, L - 1], rng.integers(0, L, 5)]))
    for h in range(H):
        a = orc.attn_vjp_dq_rows(q[0, :, h], k[0, :, h], v[0, :, h], do[0, :, h], mode, c, n,
                                 scale, rows, dlse=dlse[0, h], groups=groups, block=3)
        np.testing.assert_allclose(a, dQ[0, rows, h], rtol=1e-12, atol=1e-13)
        bk, bv = orc.attn_vjp_dkdv_cols(q[0, :, h], k[0, :, h], v[0, :, h], do[0, :, h], mode, c,
                                        n, scale, cols, dlse=dlse[0, h], groups=groups, block=4)
        np.testing.assert_allclose(bk, dK[0, cols, h], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(bv, dV[0, cols, h], rtol=1e-12, atol=1e-13)


def _golden_cases():
    import json
    import os
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "vjp_closed_form.json")
    with open(path) as f:
        return json.load(f)["cases"]


def _g(x):
    if isinstance(x, list):
        return [_g(y) for y in x]
    if isinstance(x, str):
        return float(eval(x, {"__builtins__": {}}, {"ln2": math.log(2), "ln3": math.log(3)}))
    return float(x)


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_hand_derived_cases(case):
    # tests/golden/vjp_closed_form.json: gradients derived by hand
    t = {k: np.array(_g(case[k])) for k in ("q", "k", "v", "do", "dQ", "dK", "dV")}
    dlse = np.array(_g(case["dlse"])) if "dlse" in case else None
    dQ, dK, dV = orc.attn_vjp_rows(t["q"], t["k"], t["v"], t["do"], case["mode"],
                                   case["chunk_tokens"], case["n_chunks"], case["scale"],
                                   dlse=dlse)
    np.testing.assert_allclose(dQ, t["dQ"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dK, t["dK"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(dV, t["dV"], rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Planted mistakes: each must fail at least one pin above.

def _vjp_variant(kind):
    def rows(q, k, v, do, mode, c, n, scale, dlse=None, groups=None):
        q, k, v, do = (orc._as64(x) for x in (q, k, v, do))
        L, d = q.shape
        s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
        t = np.arange(L)
        M = orc.allowed_groups(groups, t[:, None], t[None, :]) if groups is not None \
            else orc.allowed(mode, c, n, t[:, None], t[None, :])
        S = np.where(M, s * (q @ k.T), -np.inf)
        P = np.exp(S - np.logaddexp.reduce(S, axis=1)[:, None])
        dP = do @ v.T
        delta = (P * dP).sum(axis=1, keepdims=True)
        dS = P * dP if kind == "drop_delta" else P * (dP - delta)
        if dlse is not None:
            sign = -1.0 if kind == "dlse_sign" else 1.0
            dS = dS + sign * P * orc._as64(dlse)[:, None]
        dQ = (dS @ k) if kind == "dq_no_scale" else s * (dS @ k)
        dK = s * (dS @ q) if kind == "dk_not_transposed" else s * (dS.T @ q)
        dV = (P @ do) if kind == "dv_not_transposed" else P.T @ do
        return dQ, dK, dV
    return rows


PIN_CHECKS = (
    [lambda c=c: test_against_torch_reverse_autodiff(c) for c in CASES]
    + [lambda c=c: test_lse_cotangent_against_autodiff(c) for c in CASES]
    + [lambda c=c: test_adjoint_of_the_pinned_jvp(c) for c in CASES]
    + [lambda: test_finite_differences_of_a_scalar_loss(TF),
       lambda: test_finite_differences_of_a_scalar_loss(BC),
       test_one_admissible_key_per_row, test_zero_cotangent_gives_zero_gradients,
       test_lse_cotangent_on_a_zero_query]
    + [lambda c=c: test_hand_derived_cases(c) for c in _golden_cases()]
)


def _failures(monkeypatch, fn):
    monkeypatch.setattr(orc, "attn_vjp_rows", fn)
    n = 0
    for check in PIN_CHECKS:
        try:
            check()
        except AssertionError:
            n += 1
    return n


@pytest.mark.parametrize("kind", ["drop_delta", "dlse_sign", "dq_no_scale", "dk_not_transposed",
                                  "dv_not_transposed"])
def test_backward_mistakes_are_caught(monkeypatch, kind):
    assert _failures(monkeypatch, _vjp_variant(kind)) > 0


def test_correct_rewrite_is_not_flagged(monkeypatch):
    assert _failures(monkeypatch, _vjp_variant("none")) == 0
