"""Property-based pins of the oracle on random masks (hypothesis): for random
valid group tables (the general mask form: query groups with up to two key
ranges), random sizes, scales and inputs, the oracle's JVP equals forward-mode
autodiff and its backward equals reverse-mode autodiff of torch's float64
math-backend attention under the same explicit mask."""
import math

import numpy as np
import torch
import torch.nn.functional as F
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st
from torch.func import jvp
from torch.nn.attention import SDPBackend, sdpa_kernel

from oracle import attn_jvp_oracle as orc


@st.composite
def group_tables(draw):
    L = draw(st.integers(1, 12))
    cuts = sorted(set(draw(st.lists(st.integers(1, L - 1), max_size=4)) if L > 1 else []) | {L})
    groups = []
    for end in cuts:
        pts = sorted(draw(st.lists(st.integers(0, L), min_size=4, max_size=4)))
        a0, a1, b0, b1 = pts
        if a1 - a0 + b1 - b0 == 0:  # no key: give the group key 0, keep the order
            a0, a1 = 0, 1
            b0 = b1 = max(b0, 1)
        groups.append((end, a0, a1, b0, b1))
    return L, groups


def _t(x):
    return torch.from_numpy(x)[None, None]


@settings(max_examples=40, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(table=group_tables(), d=st.integers(1, 6), scale=st.sampled_from([None, 0.3, 1.7]),
       seed=st.integers(0, 2 ** 16))
def test_jvp_and_backward_match_autodiff_on_random_masks(table, d, scale, seed):
    L, groups = table
    M = orc.mask_matrix_groups(groups)
    g = np.asarray(groups)
    assert (g[:, 1] <= g[:, 2]).all() and (g[:, 2] <= g[:, 3]).all() and (g[:, 3] <= g[:, 4]).all()
    assert M.any(axis=1).all()  # every row has a key
    rng = np.random.default_rng(seed)
    q, k, v, tq, tk, tv, do = (rng.standard_normal((L, d)) for _ in range(7))
    s = 1.0 / math.sqrt(d) if scale is None else scale
    mask = torch.from_numpy(M)

    def f(a, b, c):
        with sdpa_kernel(SDPBackend.MATH):
            return F.scaled_dot_product_attention(a, b, c, attn_mask=mask, scale=s)

    O, tO, _ = orc.attn_jvp_rows(q, k, v, tq, tk, tv, 0, 1, 1, scale, np.arange(L),
                                 groups=groups)
    o_ref, to_ref = jvp(f, (_t(q), _t(k), _t(v)), (_t(tq), _t(tk), _t(tv)))
    np.testing.assert_allclose(O, o_ref[0, 0].numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(tO, to_ref[0, 0].numpy(), rtol=1e-10, atol=1e-11)

    dQ, dK, dV = orc.attn_vjp_rows(q, k, v, do, 0, 1, 1, scale, groups=groups)
    xs = [_t(a).requires_grad_(True) for a in (q, k, v)]
    f(*xs).backward(_t(do))
    for got, x in zip((dQ, dK, dV), xs):
        np.testing.assert_allclose(got, x.grad[0, 0].numpy(), rtol=1e-10, atol=1e-11)
