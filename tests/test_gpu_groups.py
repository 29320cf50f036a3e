"""GPU parity of general (group-table) masks through attn_jvp_fwd_groups.

- The teacher-forcing and block-causal masks written as group tables give the
  same bits as the {mode, c, n} form (same schedule, same arithmetic), for the
  CTA-pair kernel (d = 128), the single-CTA kernel (d = 64) and fp32.
- Other tables, shaped like the masks the pages mention (a KV-cache step that
  reads a cached prefix and its own chunk, sliding windows, dense attention,
  two ranges with gaps, one-row groups), against the oracle within the
  tolerances of the parity tests.
"""
import numpy as np
import pytest
import torch

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import inputs as wl
from oracle import attn_jvp_oracle as orc

pytestmark = pytest.mark.gpu

TF, BC = wl.TEACHER_FORCING, wl.BLOCK_CAUSAL
TOL = {"bf16": (2e-2, 1e-3), "f32": (1e-4, 1e-4)}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from attention_jvp_attn_b200 import build
    build.build()


def _inputs(B, L, H, d, dtype, seed, device):
    g = torch.Generator(device=device).manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return {n: torch.randn((B, L, H, d), generator=g, device=device).to(dt)
            for n in wl.TENSOR_ORDER}


def _run_groups(x, groups, scale=None):
    out = aj.attn_jvp_groups(*(x[n] for n in wl.TENSOR_ORDER), groups, scale)
    assert aj.sync_status() == 0
    return out


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 64)])
@pytest.mark.parametrize("mode,c,n", [(TF, 24, 5), (TF, 200, 3), (BC, 130, 3), (BC, 77, 2)])
def test_mode_tables_match_mode_form_bitwise(cuda_device, dtype, d, mode, c, n):
    L = orc.seq_len(mode, c, n)
    x = _inputs(2, L, 2, d, dtype, 300 + c + n, cuda_device)
    a = aj.attn_jvp(*(x[k] for k in wl.TENSOR_ORDER), mode, c, n)
    assert aj.sync_status() == 0
    b = _run_groups(x, orc.group_table(mode, c, n))
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.uint8), v.view(torch.uint8))


def _kv_cache_step(prefix, chunk):
    # new chunk of `chunk` tokens after a cached prefix: every new row sees the
    # prefix and its own chunk (keys [0, prefix + chunk)); prefix rows see the prefix
    L = prefix + chunk
    return [(prefix, 0, prefix, prefix, prefix), (L, 0, prefix, prefix, L)]


def _sliding(L, w, step):
    groups, r = [], 0
    while r < L:
        e = min(L, r + step)
        groups.append((e, max(0, r - w), e, e, e))
        r = e
    return groups


def _two_ranges_with_gaps(L):
    q = L // 4
    return [(q, 0, q, 2 * q, 3 * q), (2 * q, q // 2, q, 3 * q, L), (L, 0, 1, L - 5, L)]


TABLES = {
    "kv_cache_step": (_kv_cache_step(300, 170), None),
    "sliding_window": (_sliding(517, 96, 40), None),
    "dense": ([(333, 0, 333, 333, 333)], None),
    "gaps": (_two_ranges_with_gaps(640), None),
    "one_row_groups": ([(i + 1, max(0, i - 50), i + 1, min(i + 200, 260), 260) for i in range(60)]
                       + [(260, 100, 140, 140, 140)], None),
    "scaled": (_sliding(384, 128, 128), 0.05),
}


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 64)])
@pytest.mark.parametrize("name", list(TABLES))
def test_tables_against_oracle(cuda_device, dtype, d, name):
    groups, scale = TABLES[name]
    L = groups[-1][0]
    x = _inputs(1, L, 2, d, dtype, 77 + len(name), cuda_device)
    o, to, lse = _run_groups(x, groups, scale)
    xc = {k: v.cpu() for k, v in x.items()}
    O, tO, LSE = orc.attn_jvp_dense(xc["q"], xc["k"], xc["v"], xc["tq"], xc["tk"], xc["tv"],
                                    TF, 1, 1, scale, groups=groups)
    t_o, t_l = TOL[dtype]
    for nm, got, ref, tol in (("O", o, O, t_o), ("tO", to, tO, t_o), ("LSE", lse, LSE, t_l)):
        g = got.double().cpu().numpy()
        assert np.isfinite(g).all(), nm
        err = np.abs(g - ref)
        assert (err <= tol * (1.0 + np.abs(ref))).all(), (nm, float(err.max()))
