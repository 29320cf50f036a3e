"""The CTA-pair kernel (head dim 128): two SMs per 256 query rows, each holding
half of every key/value tile, with the tensor-core products issued for both.

It performs the same arithmetic in the same order as the single-CTA kernel:
the pair's key-tile schedule is the union of its two halves' schedules, and
the tiles a row cannot see contribute exact zeros. So its outputs must equal
the single-CTA kernel's bit for bit; they are also held to the oracle within
the bf16 tolerances of the parity tests.
"""
import numpy as np
import pytest
import torch

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import inputs as wl
from oracle import attn_jvp_oracle as orc

pytestmark = pytest.mark.gpu

TF, BC = wl.TEACHER_FORCING, wl.BLOCK_CAUSAL


@pytest.fixture(scope="module", autouse=True)
def _built():
    from attention_jvp_attn_b200 import build
    build.build()
    yield
    aj.set_cta_pairs(False)


def _run(w, x, pair):
    aj.set_cta_pairs(pair)
    out = aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode, w.chunk_tokens,
                      w.n_chunks, w.scale)
    assert aj.sync_status() == 0
    return out


def _assert_same_bits(a, b):
    for name, u, v in zip(("O", "tO", "LSE"), a, b):
        assert torch.equal(u.view(torch.uint8), v.view(torch.uint8)), name


CASES = [
    # (mode, c, n, B, H): odd and even numbers of 128-row tiles (a ragged last
    # pair), chunk boundaries inside a pair, several items per CTA pair
    (TF, 16, 4, 2, 3),
    (TF, 24, 5, 1, 2),
    (TF, 200, 2, 2, 1),
    (TF, 300, 1, 1, 2),
    (TF, 1, 7, 1, 1),
    (TF, 256, 4, 1, 2),
    (BC, 130, 3, 1, 3),
    (BC, 77, 1, 1, 1),
    (BC, 200, 5, 2, 2),
]


@pytest.mark.parametrize("mode,c,n,B,H", CASES)
def test_pairs_match_single_cta_and_oracle(cuda_device, mode, c, n, B, H):
    w = wl.Workload(f"pairs_{mode}_{c}_{n}", B=B, H=H, d=128, n_chunks=n, chunk_tokens=c,
                    mode=mode, seed=9000 + 7 * c + n)
    x = wl.make_inputs(w, device=cuda_device)
    single = _run(w, x, False)
    pair = _run(w, x, True)
    _assert_same_bits(single, pair)
    xc = {k: v.cpu() for k, v in x.items()}
    O, tO, LSE = orc.attn_jvp_dense(xc["q"], xc["k"], xc["v"], xc["tq"], xc["tk"], xc["tv"],
                                    w.mode, w.chunk_tokens, w.n_chunks, w.scale)
    for name, got, ref, tol in (("O", pair[0], O, 2e-2), ("tO", pair[1], tO, 2e-2),
                                ("LSE", pair[2], LSE, 1e-3)):
        g = got.double().cpu().numpy()
        assert np.isfinite(g).all(), name
        assert (np.abs(g - ref) <= tol * (1.0 + np.abs(ref))).all(), name


@pytest.mark.parametrize("name", ["framewise_tf_bf16", "block_causal_bf16"])
def test_pairs_match_single_cta_at_full_size(cuda_device, name):
    w = wl.WORKLOADS[name]
    x = wl.make_inputs(w, device=cuda_device)
    _assert_same_bits(_run(w, x, False), _run(w, x, True))


def test_pair_switch_reports_previous_setting():
    aj.set_cta_pairs(False)
    assert aj.set_cta_pairs(True) is False
    assert aj.set_cta_pairs(False) is True
