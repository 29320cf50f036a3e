"""The CTA-pair path of head dim 128: two SMs per 256 query rows, each holding
half of every key/value tile, with the tensor-core products issued for both.

Cases that only a pair has: an odd number of 128-row tiles (the last pair's
second CTA has no valid rows), chunk boundaries between the two halves of a
pair (the pair's key-tile schedule is the union of its halves', and tiles a
row cannot see contribute exact zeros), several items per pair and items with
a single key tile. Each is held to the oracle within the bf16 tolerances of
the parity tests, and a repeated call must give the same bits.
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


def _run(w, x):
    out = aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode, w.chunk_tokens,
                      w.n_chunks, w.scale)
    assert aj.sync_status() == 0
    return out


CASES = [
    # (mode, c, n, B, H)
    (TF, 16, 4, 2, 3),    # L = 128: one pair, its second CTA past the end
    (TF, 24, 5, 1, 2),    # chunk boundaries inside both halves of a pair
    (TF, 200, 2, 2, 1),   # 7 tiles: odd
    (TF, 300, 1, 1, 2),
    (TF, 1, 7, 1, 1),     # one-token chunks
    (TF, 256, 4, 1, 2),   # chunks aligned to pairs
    (TF, 128, 3, 3, 5),   # chunks aligned to tiles, not pairs; many items per pair
    (BC, 130, 3, 1, 3),
    (BC, 77, 1, 1, 1),    # a single key tile
    (BC, 200, 5, 2, 2),
]


@pytest.mark.parametrize("mode,c,n,B,H", CASES)
def test_pairs_against_oracle(cuda_device, mode, c, n, B, H):
    w = wl.Workload(f"pairs_{mode}_{c}_{n}", B=B, H=H, d=128, n_chunks=n, chunk_tokens=c,
                    mode=mode, seed=9000 + 7 * c + n)
    x = wl.make_inputs(w, device=cuda_device)
    got = _run(w, x)
    xc = {k: v.cpu() for k, v in x.items()}
    O, tO, LSE = orc.attn_jvp_dense(xc["q"], xc["k"], xc["v"], xc["tq"], xc["tk"], xc["tv"],
                                    w.mode, w.chunk_tokens, w.n_chunks, w.scale)
    for name, t, ref, tol in (("O", got[0], O, 2e-2), ("tO", got[1], tO, 2e-2),
                              ("LSE", got[2], LSE, 1e-3)):
        g = t.double().cpu().numpy()
        assert np.isfinite(g).all(), name
        assert (np.abs(g - ref) <= tol * (1.0 + np.abs(ref))).all(), name
    again = _run(w, x)
    for a, b in zip(got, again):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
