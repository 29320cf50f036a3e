"""Backward of the primal attention at the full frame-wise size (B=1, H=12,
d=128, 21 chunks of 1560 tokens, L=65520, bf16), in the launch configuration
`bench.py --backward` times: the forward kernel's O and LSE go into the
backward, as in training. The float64 oracle computes sampled outputs one by
one from the seeded inputs alone:

- dQ rows: chunk edges, the rows around 128-row tile boundaries near chunk
  boundaries, the ragged tail and seeded random rows;
- dK and dV columns: keys of the first, a middle and the last noisy chunk and
  of the last clean chunk (edges, 32- and 128-key tile boundaries, seeded
  random keys). Only one chunk of rows attends to each of those keys, so the
  oracle forms them in seconds; the last noisy chunk holds the ragged tail.

Tolerance 2e-2 (1 + |ref|), as for the small bf16 backward cases: bf16
outputs, and O and LSE from the bf16 forward.
"""
import numpy as np
import pytest
import torch

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import inputs as wl
from oracle import attn_jvp_oracle as orc

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _built():
    from attention_jvp_attn_b200 import build
    build.build()


def sample_cols(w, n_random=8, seed=3):
    c, n, L = w.chunk_tokens, w.n_chunks, w.L
    if w.mode == wl.TEACHER_FORCING:
        starts = [n * c, n * c + (n // 2) * c, n * c + (n - 1) * c, (n - 1) * c]
    else:
        starts = [(n - 1) * c]
    rng = np.random.default_rng(seed)
    cols = set()
    for a in starts:
        for off in (0, 31, 32, 127, 128, c - 1):
            if off < c:
                cols.add(a + off)
        cols.update((a + rng.integers(0, c, n_random)).tolist())
    return sorted(x for x in cols if 0 <= x < L)


def sampled_check(w, device, heads):
    x = wl.make_inputs(w, device=device)
    o, _, lse = aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode,
                            w.chunk_tokens, w.n_chunks, w.scale)
    g = torch.Generator(device=device).manual_seed(1234)
    do = torch.randn(x["q"].shape, generator=g, device=device).to(x["q"].dtype)
    dq, dk, dv = aj.attn_jvp_bwd(x["q"], x["k"], x["v"], o, do, lse, w.mode, w.chunk_tokens,
                                 w.n_chunks, w.scale)
    assert aj.sync_status() == 0
    rows = wl.sample_rows(w, n_random=64, max_rows=192)
    cols = sample_cols(w)
    m = (w.mode, w.chunk_tokens, w.n_chunks, w.scale)
    for h in heads:
        sl = [t[0, :, h].cpu() for t in (x["q"], x["k"], x["v"], do)]
        ref_q = orc.attn_vjp_dq_rows(*sl, *m, rows)
        ref_k, ref_v = orc.attn_vjp_dkdv_cols(*sl, *m, cols)
        for name, got, ref in (("dQ", dq[0, rows, h], ref_q), ("dK", dk[0, cols, h], ref_k),
                               ("dV", dv[0, cols, h], ref_v)):
            a = got.double().cpu().numpy()
            err = np.abs(a - ref)
            assert np.isfinite(a).all() and (err <= TOL * (1.0 + np.abs(ref))).all(), \
                (name, h, float(err.max()))


def test_framewise_backward_sampled(cuda_device):
    sampled_check(wl.FRAMEWISE_TF, cuda_device, heads=(wl.FRAMEWISE_TF.H - 1,))
