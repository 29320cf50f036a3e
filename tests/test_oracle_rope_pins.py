"""Pins of the oracle's rotary position embedding (rope_rotate) and of the
attention JVP with RoPE in front (attn_jvp_rope_dense), against values that do
not come from those functions:

- closed forms: zero angles leave x unchanged; a quarter turn maps each pair
  (a, b) to (-b, a); a half turn negates;
- the rotation preserves the norm of every pair, and turning by phi then by
  -phi gives x back;
- the relative-position property of 1-D RoPE: (R_m q) . (R_n k) depends only
  on n - m;
- a complex-number restatement in torch (pairs as complex numbers times
  e^{i phi}), and forward-mode autodiff of that restatement composed with
  torch's math-backend attention under the mask, for O and tO.

Planted mistakes at the end (pairs i and i + d/2 instead of adjacent pairs, a
wrong sign of sin, tangents left unrotated) must each fail a pin.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
from torch.func import jvp
from torch.nn.attention import SDPBackend, sdpa_kernel

from oracle import attn_jvp_oracle as orc

TF, BC = orc.TEACHER_FORCING, orc.BLOCK_CAUSAL


def _x(L, H, d, seed):
    return np.random.default_rng(seed).standard_normal((1, L, H, d))


def _angles(L, d, seed):
    phi = np.random.default_rng(seed).uniform(-4.0, 4.0, (L, d // 2))
    return np.cos(phi), np.sin(phi)


def test_zero_angles_are_the_identity():
    x = _x(5, 2, 8, 1)
    c, s = np.ones((5, 4)), np.zeros((5, 4))
    np.testing.assert_array_equal(orc.rope_rotate(x, c, s), x)


def test_quarter_and_half_turns():
    x = _x(3, 1, 6, 2)
    q = orc.rope_rotate(x, np.zeros((3, 3)), np.ones((3, 3)))  # phi = pi/2
    np.testing.assert_array_equal(q[..., 0::2], -x[..., 1::2])
    np.testing.assert_array_equal(q[..., 1::2], x[..., 0::2])
    h = orc.rope_rotate(x, -np.ones((3, 3)), np.zeros((3, 3)))  # phi = pi
    np.testing.assert_array_equal(h, -x)


def test_one_pair_by_hand():
    # (3, 4) turned by phi with cos = 0.6, sin = 0.8: (3*0.6 - 4*0.8, 3*0.8 + 4*0.6)
    x = np.array([3.0, 4.0]).reshape(1, 1, 1, 2)
    y = orc.rope_rotate(x, np.array([[0.6]]), np.array([[0.8]]))
    np.testing.assert_allclose(y.ravel(), [-1.4, 4.8], rtol=0, atol=1e-15)


def test_pair_norms_and_inverse():
    L, d = 7, 16
    x = _x(L, 3, d, 3)
    c, s = _angles(L, d, 4)
    y = orc.rope_rotate(x, c, s)
    np.testing.assert_allclose(y[..., 0::2] ** 2 + y[..., 1::2] ** 2,
                               x[..., 0::2] ** 2 + x[..., 1::2] ** 2, rtol=1e-13)
    np.testing.assert_allclose(orc.rope_rotate(y, c, -s), x, rtol=0, atol=1e-13)


def test_relative_position_property():
    L, d = 12, 8
    cos, sin = orc.rope_angles_1d(L, d)
    rng = np.random.default_rng(5)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    X = np.broadcast_to(q, (1, L, 1, d)).copy()
    Y = np.broadcast_to(k, (1, L, 1, d)).copy()
    Rq, Rk = orc.rope_rotate(X, cos, sin)[0, :, 0], orc.rope_rotate(Y, cos, sin)[0, :, 0]
    G = Rq @ Rk.T  # G[m, n] = (R_m q) . (R_n k)
    for delta in range(-L + 1, L):
        vals = np.diagonal(G, offset=delta)
        np.testing.assert_allclose(vals, vals[0], rtol=1e-12, atol=1e-12)
    # and it is not constant across offsets (the positions matter)
    assert np.ptp([G[0, j] for j in range(L)]) > 1e-3


def _torch_rope(x, cos, sin):
    """Pairs as complex numbers multiplied by e^{i phi} ([1, H, L, d] layout)."""
    z = torch.view_as_complex(x.reshape(*x.shape[:-1], -1, 2).contiguous())
    rot = torch.polar(torch.ones_like(cos), torch.atan2(sin, cos))[None, None]
    return torch.view_as_real(z * rot).reshape(x.shape)


def test_complex_restatement():
    L, H, d = 9, 2, 12
    x = _x(L, H, d, 6)
    c, s = _angles(L, d, 7)
    ref = _torch_rope(torch.from_numpy(x).permute(0, 2, 1, 3), torch.from_numpy(c),
                      torch.from_numpy(s)).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(orc.rope_rotate(x, c, s), ref, rtol=0, atol=1e-13)


@pytest.mark.parametrize("mode,cc,n,d", [(TF, 2, 3, 8), (BC, 3, 3, 6)])
def test_rope_attention_jvp_against_autodiff(mode, cc, n, d):
    L, H = orc.seq_len(mode, cc, n), 2
    q, k, v, tq, tk, tv = (_x(L, H, d, 10 + i) for i in range(6))
    c, s = _angles(L, d, 8)
    O, tO, _ = orc.attn_jvp_rope_dense(q, k, v, tq, tk, tv, c, s, mode, cc, n)
    mask = torch.from_numpy(orc.mask_matrix(mode, cc, n))
    C, S = torch.from_numpy(c), torch.from_numpy(s)
    T = lambda a: torch.from_numpy(a).permute(0, 2, 1, 3)

    def f(a, b, w):
        with sdpa_kernel(SDPBackend.MATH):
            return F.scaled_dot_product_attention(_torch_rope(a, C, S), _torch_rope(b, C, S), w,
                                                  attn_mask=mask, scale=1.0 / math.sqrt(d))

    o_ref, to_ref = jvp(f, (T(q), T(k), T(v)), (T(tq), T(tk), T(tv)))
    back = lambda t: t.permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(O, back(o_ref), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(tO, back(to_ref), rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------
# Planted mistakes

def _rope_half_pairs(x, cos, sin):
    x = orc._as64(x)
    h = x.shape[-1] // 2
    c, s = orc._as64(cos)[None, :, None, :], orc._as64(sin)[None, :, None, :]
    a, b = x[..., :h], x[..., h:]
    return np.concatenate([a * c - b * s, a * s + b * c], axis=-1)


def _rope_sin_sign(x, cos, sin):
    return orc.rope_rotate.__wrapped__(x, cos, -orc._as64(sin))


def _jvp_rope_unrotated_tangents(q, k, v, tq, tk, tv, cos, sin, mode, c, n, scale=None,
                                 groups=None):
    R = orc.rope_rotate
    return orc.attn_jvp_dense(R(q, cos, sin), R(k, cos, sin), v, tq, tk, tv, mode, c, n, scale,
                              groups=groups)


PIN_CHECKS = [
    test_zero_angles_are_the_identity, test_quarter_and_half_turns, test_one_pair_by_hand,
    test_pair_norms_and_inverse, test_relative_position_property, test_complex_restatement,
    lambda: test_rope_attention_jvp_against_autodiff(TF, 2, 3, 8),
    lambda: test_rope_attention_jvp_against_autodiff(BC, 3, 3, 6),
]


def _failures(monkeypatch, attr, fn):
    monkeypatch.setattr(orc, attr, fn)
    n = 0
    for check in PIN_CHECKS:
        try:
            check()
        except AssertionError:
            n += 1
    return n


@pytest.mark.parametrize("attr,mutant", [
    ("rope_rotate", _rope_half_pairs),
    ("rope_rotate", _rope_sin_sign),
    ("attn_jvp_rope_dense", _jvp_rope_unrotated_tangents),
])
def test_rope_mistakes_are_caught(monkeypatch, attr, mutant):
    _rope_sin_sign.__wrapped__ = orc.rope_rotate
    assert _failures(monkeypatch, attr, mutant) > 0


def test_unmutated_oracle_passes_every_pin():
    for check in PIN_CHECKS:
        check()
