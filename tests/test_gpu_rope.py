"""GPU parity of the rotary position embedding (attn_jvp_rope) with the
float64 oracle, and of RoPE followed by the attention JVP (attn_jvp_rope).

- The rotation alone, element by element: the kernel computes in fp32 from
  the exact inputs and rounds to the output type, so
  |err| <= u |ref| + 1e-6 (|x_2i| + |x_2i+1|), u = 2^-8 for bf16 and 2^-24 for
  fp32. Cases: both dtypes, d = 64 and 128, random angles and 1-D positions,
  odd L, B > 1.
- In place (outputs = inputs) gives the same bits as out of place.
- RoPE then attention, against attn_jvp_rope_dense: the forward's tolerances
  (2e-2 (1+|ref|) for bf16 O and tO, 1e-4 for fp32). LSE is held to 2e-3 for
  bf16: the rotated q and k are rounded to bf16 before the attention (2^-8
  relative per element), which moves the logits by up to ~2^-8 |S|.
"""
import numpy as np
import pytest
import torch

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import inputs as wl
from oracle import attn_jvp_oracle as orc

pytestmark = pytest.mark.gpu

TF, BC = wl.TEACHER_FORCING, wl.BLOCK_CAUSAL
U = {"bf16": 2.0 ** -8, "f32": 2.0 ** -24}


@pytest.fixture(scope="module", autouse=True)
def _built():
    from attention_jvp_attn_b200 import build
    build.build()


def _tensors(B, L, H, d, dtype, seed, device, n=4, std=1.0):
    g = torch.Generator(device=device).manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    return [(torch.randn((B, L, H, d), generator=g, device=device) * std).to(dt) for _ in range(n)]


def _angles(L, d, kind, seed):
    if kind == "random":
        phi = np.random.default_rng(seed).uniform(-np.pi, np.pi, (L, d // 2))
        c, s = np.cos(phi), np.sin(phi)
    else:
        c, s = orc.rope_angles_1d(L, d)
    return c.astype(np.float32), s.astype(np.float32)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("f32", 64), ("f32", 128)])
@pytest.mark.parametrize("B,L,kind", [(1, 333, "random"), (2, 96, "1d"), (1, 1, "random")])
def test_rotation_against_oracle(cuda_device, dtype, d, B, L, kind):
    xs = _tensors(B, L, 3, d, dtype, 10 + L + d, cuda_device)
    c, s = _angles(L, d, kind, L)
    cd, sd = torch.from_numpy(c).to(cuda_device), torch.from_numpy(s).to(cuda_device)
    out = aj.rope(*xs, cd, sd)
    assert aj.sync_status() == 0
    for x, y in zip(xs, out):
        xc = x.double().cpu().numpy()
        ref = orc.rope_rotate(xc, c, s)
        pair = np.repeat(np.abs(xc[..., 0::2]) + np.abs(xc[..., 1::2]), 2, axis=-1)
        got = y.double().cpu().numpy()
        assert (np.abs(got - ref) <= U[dtype] * np.abs(ref) + 1e-6 * pair).all()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_in_place_matches_out_of_place(cuda_device, dtype):
    L, d = 250, 128
    xs = _tensors(2, L, 2, d, dtype, 3, cuda_device)
    c, s = _angles(L, d, "random", 4)
    cd, sd = torch.from_numpy(c).to(cuda_device), torch.from_numpy(s).to(cuda_device)
    a = aj.rope(*xs, cd, sd)
    b = [x.clone() for x in xs]
    aj.rope(*b, cd, sd, out=tuple(b))
    assert aj.sync_status() == 0
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("dtype,d,mode,c,n", [("bf16", 128, TF, 100, 3), ("bf16", 64, BC, 130, 3),
                                              ("f32", 64, TF, 24, 5)])
def test_rope_then_attention_against_oracle(cuda_device, dtype, d, mode, c, n):
    L = orc.seq_len(mode, c, n)
    r2 = 2 ** -0.5
    q, k, tq, tk = _tensors(1, L, 2, d, dtype, 40 + d, cuda_device, std=r2)
    v, tv = _tensors(1, L, 2, d, dtype, 41 + d, cuda_device, n=2)
    cs, sn = _angles(L, d, "random", 5)
    cd, sd = torch.from_numpy(cs).to(cuda_device), torch.from_numpy(sn).to(cuda_device)
    o, to, lse = aj.attn_jvp_rope(q, k, v, tq, tk, tv, cd, sd, mode, c, n)
    assert aj.sync_status() == 0
    cpu = [t.cpu() for t in (q, k, v, tq, tk, tv)]
    O, tO, LSE = orc.attn_jvp_rope_dense(*cpu, cs, sn, mode, c, n)
    t_o = 2e-2 if dtype == "bf16" else 1e-4
    t_l = 2e-3 if dtype == "bf16" else 1e-4
    for name, got, ref, tol in (("O", o, O, t_o), ("tO", to, tO, t_o), ("LSE", lse, LSE, t_l)):
        g = got.double().cpu().numpy()
        err = np.abs(g - ref)
        assert np.isfinite(g).all() and (err <= tol * (1.0 + np.abs(ref))).all(), \
            (name, float(err.max()))
