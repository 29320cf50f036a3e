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


# ---- the rotation and the attention in one call -------------------------------------------
# attn_jvp_rope runs the rotation phase and the attention in one kernel launch
# for bf16 (the CTAs meet at a grid barrier in between). Both halves compute
# exactly what the separate rotation pass and attn_jvp compute, so the fused
# call must give the same bits: the four rotated tensors, O, tO and LSE.

@pytest.mark.parametrize("dtype,d,mode,c,n,B", [
    ("bf16", 128, TF, 150, 3, 1),   # CTA pairs, ragged last 256-row block
    ("bf16", 64, TF, 100, 4, 2),    # single CTAs, B = 2
    ("bf16", 128, BC, 1560, 2, 1),  # longer chunks
    ("bf16", 64, BC, 7, 5, 1),      # chunks shorter than a tile, L = 35
    ("f32", 64, TF, 40, 2, 1),      # fp32: rotation pass, then the CUDA-core kernel
])
def test_fused_rope_equals_rotation_then_attention(cuda_device, dtype, d, mode, c, n, B):
    L = orc.seq_len(mode, c, n)
    H = 3
    q, k, v, tq, tk, tv = _tensors(B, L, H, d, dtype, 70 + L + d, cuda_device, n=6)
    cs, sn = _angles(L, d, "random", L + d)
    cd, sd = torch.from_numpy(cs).to(cuda_device), torch.from_numpy(sn).to(cuda_device)
    (o, to, lse), rot = aj.attn_jvp_rope(q, k, v, tq, tk, tv, cd, sd, mode, c, n,
                                         return_rotated=True)
    assert aj.sync_status() == 0
    ref_rot = aj.rope(q, k, tq, tk, cd, sd)
    ref = aj.attn_jvp(ref_rot[0], ref_rot[1], v, ref_rot[2], ref_rot[3], tv, mode, c, n)
    assert aj.sync_status() == 0
    for got, want in zip(rot + (o, to, lse), tuple(ref_rot) + tuple(ref)):
        assert torch.equal(got.view(torch.uint8), want.view(torch.uint8))


def test_fused_rope_in_place_and_repeated(cuda_device):
    # rotated buffers = the inputs (in place); the next call, on the rotated
    # tensors' originals again, uses the next grid-barrier word
    B, L, H, d, mode, c, n = 1, 600, 2, 128, TF, 100, 3
    q, k, v, tq, tk, tv = _tensors(B, L, H, d, "bf16", 5, cuda_device, n=6)
    cs, sn = _angles(L, d, "random", 9)
    cd, sd = torch.from_numpy(cs).to(cuda_device), torch.from_numpy(sn).to(cuda_device)
    first = aj.attn_jvp_rope(q, k, v, tq, tk, tv, cd, sd, mode, c, n)
    ins = [t.clone() for t in (q, k, tq, tk)]
    second = aj.attn_jvp_rope(ins[0], ins[1], v, ins[2], ins[3], tv, cd, sd, mode, c, n,
                              rotated=tuple(ins))
    assert aj.sync_status() == 0
    ref_rot = aj.rope(q, k, tq, tk, cd, sd)
    for a, b in zip(first, second):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    for got, want in zip(ins, ref_rot):
        assert torch.equal(got.view(torch.uint8), want.view(torch.uint8))
