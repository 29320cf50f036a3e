"""GPU parity of the backward of the primal attention (attn_jvp_bwd) with the
float64 oracle's VJP, on the same seeded inputs.

The kernel takes the forward's O and LSE as inputs. The parity cases give it
the oracle's O (rounded to the input dtype) and LSE (rounded to fp32), so the
comparison isolates the backward; one case feeds it the forward kernel's own
O and LSE. Cases span ragged tails (L not a multiple of the 32-row blocks),
chunks smaller and larger than a block, both masks, group tables, both head
dims, both dtypes, an LSE cotangent and a custom scale.

Tolerances: fp32, |err| <= 1e-4 (1 + |ref|) (fp32 sums of at most a few
thousand terms). bf16, 2e-2 (1 + |ref|): the outputs are rounded to bf16
(2^-9 relative) and D_i = dO_i . O_i uses the bf16-rounded O.
"""
import numpy as np
import pytest
import torch

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import inputs as wl
from oracle import attn_jvp_oracle as orc

pytestmark = pytest.mark.gpu

TF, BC = wl.TEACHER_FORCING, wl.BLOCK_CAUSAL
TOL = {"bf16": 2e-2, "f32": 1e-4}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from attention_jvp_attn_b200 import build
    build.build()


def _sliding(L, w, step):
    groups, r = [], 0
    while r < L:
        e = min(L, r + step)
        groups.append((e, max(0, r - w), e, e, e))
        r = e
    return groups


def _inputs(B, L, H, d, dtype, seed, device, with_dlse):
    g = torch.Generator(device=device).manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = {n: torch.randn((B, L, H, d), generator=g, device=device).to(dt)
         for n in ("q", "k", "v", "do")}
    x["dlse"] = torch.randn((B, H, L), generator=g, device=device) if with_dlse else None
    return x


def _oracle_forward(xc, mask, scale):
    if isinstance(mask, list):
        return orc.attn_forward_dense(xc["q"], xc["k"], xc["v"], TF, 1, 1, scale, groups=mask)
    return orc.attn_forward_dense(xc["q"], xc["k"], xc["v"], *mask, scale)


def _oracle_vjp(xc, mask, scale, dlse):
    if isinstance(mask, list):
        return orc.attn_vjp_dense(xc["q"], xc["k"], xc["v"], xc["do"], TF, 1, 1, scale,
                                  dlse=dlse, groups=mask)
    return orc.attn_vjp_dense(xc["q"], xc["k"], xc["v"], xc["do"], *mask, scale, dlse=dlse)


def _run(x, o, lse, mask, scale):
    if isinstance(mask, list):
        out = aj.attn_jvp_bwd_groups(x["q"], x["k"], x["v"], o, x["do"], lse, mask, scale,
                                     dlse=x["dlse"])
    else:
        out = aj.attn_jvp_bwd(x["q"], x["k"], x["v"], o, x["do"], lse, *mask, scale,
                              dlse=x["dlse"])
    assert aj.sync_status() == 0
    return out


def _check(got, ref, tol):
    for name, g, r in zip(("dQ", "dK", "dV"), got, ref):
        a = g.double().cpu().numpy()
        assert np.isfinite(a).all(), name
        err = np.abs(a - r)
        assert (err <= tol * (1.0 + np.abs(r))).all(), (name, float(err.max()))


CASES = {  # dtype, d, mask ((mode, c, n) or a group table), scale, dLSE
    "tf_c24_bf16_d64": ("bf16", 64, (TF, 24, 5), None, False),
    "tf_c200_bf16_d128": ("bf16", 128, (TF, 200, 3), None, False),
    "bc_c130_bf16_d128_dlse": ("bf16", 128, (BC, 130, 3), None, True),
    "bc_c77_f32_d64": ("f32", 64, (BC, 77, 2), None, False),
    "tf_c40_f32_d128_dlse": ("f32", 128, (TF, 40, 4), None, True),
    "tf_c1_f32_d64": ("f32", 64, (TF, 1, 37), None, False),
    "sliding_bf16_d128": ("bf16", 128, _sliding(517, 96, 40), None, False),
    "kvcache_f32_d64": ("f32", 64, [(300, 0, 300, 300, 300), (470, 0, 300, 300, 470)], None,
                        True),
    "scaled_bf16_d64": ("bf16", 64, (TF, 33, 3), 0.05, False),
    # bf16 below the tensor-core path's minimum length (L = 3): CUDA-core kernels
    "short_bf16_d64": ("bf16", 64, (BC, 1, 3), None, True),
    # tensor-core path: several 128-key blocks and query tiles, ragged tail,
    # chunk edges inside tiles, group table with a gap inside a query block
    "tf_c300_bf16_d64_dlse": ("bf16", 64, (TF, 300, 2), None, True),
    "gapped_bf16_d128": ("bf16", 128, [(200, 0, 100, 300, 400), (400, 50, 250, 250, 400)], None,
                         False),
}


@pytest.mark.parametrize("name", list(CASES))
def test_backward_against_oracle(cuda_device, name):
    dtype, d, mask, scale, with_dlse = CASES[name]
    L = mask[-1][0] if isinstance(mask, list) else orc.seq_len(*mask)
    x = _inputs(2, L, 2, d, dtype, 500 + L + d, cuda_device, with_dlse)
    xc = {k: (v.cpu() if v is not None else None) for k, v in x.items()}
    O, LSE = _oracle_forward(xc, mask, scale)
    o = torch.from_numpy(O).to(device=cuda_device, dtype=x["q"].dtype).contiguous()
    lse = torch.from_numpy(LSE).to(device=cuda_device, dtype=torch.float32).contiguous()
    got = _run(x, o, lse, mask, scale)
    dlse = xc["dlse"].double().numpy() if with_dlse else None
    _check(got, _oracle_vjp(xc, mask, scale, dlse), TOL[dtype])


def test_backward_from_the_forward_kernel(cuda_device):
    # O and LSE from attn_jvp itself (bf16, d = 128, CTA-pair kernel)
    mode, c, n = TF, 90, 4
    L = orc.seq_len(mode, c, n)
    x = _inputs(1, L, 2, 128, "bf16", 71, cuda_device, False)
    t = torch.zeros_like(x["q"])
    o, _, lse = aj.attn_jvp(x["q"], x["k"], x["v"], t, t, t, mode, c, n)
    assert aj.sync_status() == 0
    got = _run(x, o, lse, (mode, c, n), None)
    xc = {k: (v.cpu() if v is not None else None) for k, v in x.items()}
    _check(got, _oracle_vjp(xc, (mode, c, n), None, None), TOL["bf16"])


def test_backward_repeats_bit_for_bit(cuda_device):
    mode, c, n = BC, 64, 5
    L = orc.seq_len(mode, c, n)
    x = _inputs(1, L, 3, 64, "bf16", 5, cuda_device, True)
    xc = {k: (v.cpu() if v is not None else None) for k, v in x.items()}
    O, LSE = _oracle_forward(xc, (mode, c, n), None)
    o = torch.from_numpy(O).to(device=cuda_device, dtype=torch.bfloat16)
    lse = torch.from_numpy(LSE).to(device=cuda_device, dtype=torch.float32)
    a = _run(x, o, lse, (mode, c, n), None)
    b = _run(x, o, lse, (mode, c, n), None)
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.int16), v.view(torch.int16))


def test_keys_no_row_attends_get_zero_gradients(cuda_device):
    # group table whose rows never look at keys [40, 64): dK, dV there are 0
    groups = [(32, 0, 20, 20, 20), (64, 0, 40, 40, 40)]
    x = _inputs(1, 64, 2, 64, "f32", 9, cuda_device, False)
    xc = {k: (v.cpu() if v is not None else None) for k, v in x.items()}
    O, LSE = _oracle_forward(xc, groups, None)
    o = torch.from_numpy(O).to(device=cuda_device, dtype=torch.float32)
    lse = torch.from_numpy(LSE).to(device=cuda_device, dtype=torch.float32)
    dq, dk, dv = _run(x, o, lse, groups, None)
    assert not dk[:, 40:].any() and not dv[:, 40:].any()
    _check((dq, dk, dv), _oracle_vjp(xc, groups, None, None), TOL["f32"])
