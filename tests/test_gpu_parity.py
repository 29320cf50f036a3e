"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on
the same seeded inputs.

Tolerances: |gpu - ref| <= 2e-2 (1 + |ref|) for O and tO in bf16 (P and U are
rounded to bf16 before their tensor-core products), <= 1e-4 (1 + |ref|) in
fp32; LSE is computed in fp32 from exact bf16 products, so it is held to
1e-3 (1 + |ref|) in bf16 and 1e-4 (1 + |ref|) in fp32.
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


def _close(name, got, ref, tol):
    got = np.asarray(got, dtype=np.float64)
    err = np.abs(got - ref)
    bound = tol * (1.0 + np.abs(ref))
    bad = err > bound
    assert np.isfinite(got).all(), f"{name}: non-finite output"
    assert not bad.any(), (f"{name}: {bad.sum()} of {bad.size} outside tolerance, "
                           f"max err {err.max():.3e}, max err/bound {(err / bound).max():.3f}")
    return float((err / bound).max())


def _run(w, x):
    o, to, lse = aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode,
                             w.chunk_tokens, w.n_chunks, w.scale)
    assert aj.sync_status() == 0
    return o, to, lse


def _dense_check(w, device):
    x = wl.make_inputs(w, device=device)
    o, to, lse = _run(w, x)
    xc = {k: v.cpu() for k, v in x.items()}
    O, tO, LSE = orc.attn_jvp_dense(xc["q"], xc["k"], xc["v"], xc["tq"], xc["tk"], xc["tv"],
                                    w.mode, w.chunk_tokens, w.n_chunks, w.scale)
    t_o, t_l = TOL[w.dtype]
    _close("O", o.double().cpu().numpy(), O, t_o)
    _close("tO", to.double().cpu().numpy(), tO, t_o)
    _close("LSE", lse.double().cpu().numpy(), LSE, t_l)


def test_tiny_fp32_teacher_forcing(cuda_device):
    _dense_check(wl.TINY_F32, cuda_device)


SMALL = [
    # (mode, c, n, d, B, H): several tiles, chunk boundaries inside tiles, ragged tails
    (TF, 16, 4, 64, 1, 2),
    (TF, 16, 4, 128, 2, 3),
    (TF, 24, 5, 128, 1, 2),
    (TF, 130, 3, 64, 1, 2),
    (TF, 200, 2, 128, 2, 1),
    (TF, 1, 7, 64, 1, 1),
    (TF, 300, 1, 128, 1, 2),
    (BC, 16, 4, 64, 2, 2),
    (BC, 130, 3, 128, 1, 3),
    (BC, 200, 4, 64, 1, 2),
    (BC, 77, 1, 128, 1, 1),
]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("mode,c,n,d,B,H", SMALL)
def test_small_dense(cuda_device, dtype, mode, c, n, d, B, H):
    w = wl.Workload(f"small_{mode}_{c}_{n}_{d}", B=B, H=H, d=d, n_chunks=n, chunk_tokens=c,
                    mode=mode, dtype=dtype, seed=c * 100 + n * 10 + d + mode)
    _dense_check(w, cuda_device)


def _rounding_bound(x, w):
    """First-order error bound of the bf16 path, per output element, from the
    bf16 rounding (unit 2^-9) of P and U = P s tS before their tensor-core
    products and of the outputs: for O, 2^-9 (sum_j P|v| + |O|); for tO,
    2^-9 (2 sum_j P|tS||v| + sum_j P|tv| + (sum_j P|tS|)|O| + |mu| sum_j P|v| + |tO|)."""
    q, k, v, tq, tk, tv = (x[n][0].double().cpu().numpy() for n in wl.TENSOR_ORDER)
    s = w.softmax_scale
    M = orc.mask_matrix(w.mode, w.chunk_tokens, w.n_chunks)
    bO = np.empty(q.shape)
    btO = np.empty(q.shape)
    for h in range(q.shape[1]):
        S = np.where(M, s * q[:, h] @ k[:, h].T, -np.inf)
        P = np.exp(S - S.max(axis=1, keepdims=True))
        P /= P.sum(axis=1, keepdims=True)
        tS = np.where(M, s * (tq[:, h] @ k[:, h].T + q[:, h] @ tk[:, h].T), 0.0)
        O = P @ v[:, h]
        mu = (P * tS).sum(axis=1, keepdims=True)
        tO = (P * (tS - mu)) @ v[:, h] + P @ tv[:, h]
        av, atv = np.abs(v[:, h]), np.abs(tv[:, h])
        bO[:, h] = P @ av + np.abs(O)
        btO[:, h] = (2 * (P * np.abs(tS)) @ av + P @ atv
                     + (P * np.abs(tS)).sum(axis=1, keepdims=True) * np.abs(O)
                     + np.abs(mu) * (P @ av) + np.abs(tO))
    u = 2.0 ** -9
    return u * bO, u * btO


def test_small_custom_scale_and_distributions(cuda_device):
    # Outside the configs' distributions (peaked softmax, large tangents) the
    # bf16 rounding of P and U dominates; hold the kernel to twice the
    # first-order bound of that rounding (plus fp32 accumulation slack).
    w = wl.Workload("scaled", B=1, H=2, d=128, n_chunks=3, chunk_tokens=100, mode=TF,
                    stds=(1.5, 1.5, 1.0, 2.0, 0.5, 1.0), scale=0.2, seed=77)
    x = wl.make_inputs(w, device=cuda_device)
    o, to, lse = _run(w, x)
    xc = {k: v.cpu() for k, v in x.items()}
    O, tO, LSE = orc.attn_jvp_dense(xc["q"], xc["k"], xc["v"], xc["tq"], xc["tk"], xc["tv"],
                                    w.mode, w.chunk_tokens, w.n_chunks, w.scale)
    bO, btO = _rounding_bound(x, w)
    for name, got, ref, b in (("O", o, O, bO), ("tO", to, tO, btO)):
        err = np.abs(got.double().cpu().numpy()[0] - ref[0])
        tol = 2.0 * b + 1e-3 * (1.0 + np.abs(ref[0]))
        assert (err <= tol).all(), f"{name}: max err/tol {(err / tol).max():.3f}"
    _close("LSE", lse.double().cpu().numpy(), LSE, TOL["bf16"][1])


def _sampled_check(w, device, heads=(0, -1), n_random=256, max_rows=None):
    x = wl.make_inputs(w, device=device)
    o, to, lse = _run(w, x)
    rows = wl.sample_rows(w, n_random=n_random, max_rows=max_rows)
    t_o, t_l = TOL[w.dtype]
    worst = 0.0
    for b in sorted({0, w.B - 1}):
        for h in sorted({hh % w.H for hh in heads}):
            sl = {k: v[b, :, h].cpu() for k, v in x.items()}
            O, tO, LSE = orc.attn_jvp_rows(sl["q"], sl["k"], sl["v"], sl["tq"], sl["tk"], sl["tv"],
                                           w.mode, w.chunk_tokens, w.n_chunks, w.scale, rows)
            idx = torch.tensor(rows, device=o.device)
            worst = max(worst, _close(f"O[{b},:,{h}]", o[b, idx, h].double().cpu().numpy(), O, t_o))
            worst = max(worst, _close(f"tO[{b},:,{h}]", to[b, idx, h].double().cpu().numpy(), tO, t_o))
            worst = max(worst, _close(f"LSE[{b},{h}]", lse[b, h, idx].double().cpu().numpy(), LSE, t_l))
    del x, o, to, lse
    torch.cuda.empty_cache()
    return worst


@pytest.mark.parametrize("w", [wl.FRAMEWISE_TF, wl.CHUNKWISE_TF, wl.BLOCK_CAUSAL_BF16],
                         ids=lambda w: w.name)
def test_full_size_sampled_rows(cuda_device, w):
    _sampled_check(w, cuda_device)


@pytest.mark.parametrize("w", wl.sweep_points(), ids=lambda w: w.name)
def test_sweep_sampled_rows(cuda_device, w):
    _sampled_check(w, cuda_device, heads=(5,), n_random=32, max_rows=256)


def test_deterministic(cuda_device):
    w = wl.Workload("det", B=1, H=4, d=128, n_chunks=5, chunk_tokens=300, mode=TF, seed=3)
    x = wl.make_inputs(w, device=cuda_device)
    a = _run(w, x)
    b = _run(w, x)
    for u, v in zip(a, b):
        assert torch.equal(u, v)


@pytest.mark.parametrize("H,d,dtype", [(2, 128, "bf16"), (5, 64, "bf16"), (12, 128, "bf16"),
                                        (3, 64, "f32")])
def test_host_buffer_entry_point(cuda_device, H, d, dtype):
    # heads go in chunks through two staging slots (5 heads: chunks of 2, 2, 1);
    # the result must be the device entry point's, bit for bit
    w = wl.Workload("host", B=2, H=H, d=d, n_chunks=3, chunk_tokens=70, mode=TF, seed=9 + H,
                    dtype=dtype)
    x = wl.make_inputs(w, device="cpu")
    xh = {k: v.pin_memory() for k, v in x.items()}
    B, L, H, d = w.B, w.L, w.H, w.d
    dt = x["q"].dtype
    out = (torch.empty((B, L, H, d), dtype=dt).pin_memory(),
           torch.empty((B, L, H, d), dtype=dt).pin_memory(),
           torch.empty((B, H, L), dtype=torch.float32).pin_memory())
    staging = torch.empty(aj.host_staging_bytes(B, L, H, d, dt), dtype=torch.uint8,
                          device=cuda_device)
    aj.attn_jvp_host(xh["q"], xh["k"], xh["v"], xh["tq"], xh["tk"], xh["tv"], w.mode,
                     w.chunk_tokens, w.n_chunks, staging, out)
    xd = {k: v.to(cuda_device) for k, v in x.items()}
    o, to, lse = _run(w, xd)
    assert torch.equal(out[0], o.cpu()) and torch.equal(out[1], to.cpu())
    assert torch.equal(out[2], lse.cpu())


def test_zero_query_tangent_matches_p_tv(cuda_device):
    # tq = tk = 0: tO must equal the primal output with v replaced by tv.
    w = wl.Workload("pt", B=1, H=2, d=128, n_chunks=4, chunk_tokens=150, mode=TF, seed=12)
    x = wl.make_inputs(w, device=cuda_device)
    z = torch.zeros_like(x["q"])
    _, to, _ = aj.attn_jvp(x["q"], x["k"], x["v"], z, z, x["tv"], TF, 150, 4)
    o2, _, _ = aj.attn_jvp(x["q"], x["k"], x["tv"], z, z, x["tv"], TF, 150, 4)
    assert aj.sync_status() == 0
    diff = (to.float() - o2.float()).abs().max().item()
    assert diff <= 2e-2, diff


def test_rejects_wrong_inputs_before_launch(cuda_device):
    w = wl.Workload("bad", B=1, H=2, d=64, n_chunks=2, chunk_tokens=16, mode=TF, seed=1)
    x = wl.make_inputs(w, device=cuda_device)
    with pytest.raises(aj.AttnJvpError) as e:
        aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], TF, 16, 3)
    assert e.value.code == 1
    q = x["q"].half()
    with pytest.raises(TypeError):
        aj.attn_jvp(q, q, q, q, q, q, TF, 16, 2)
    assert aj.sync_status() == 0
