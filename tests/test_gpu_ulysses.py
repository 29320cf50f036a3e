"""The Ulysses path on a GPU with the library's kernels as the local attention
and backward (NCCL process group of one rank: the exchange is the identity,
the kernels and the layout code are the real ones). Its outputs must equal a
direct call's, bit for bit, and the float64 oracle's within the parity
tolerances. The exchange across several ranks, with these kernels inside it,
is tested in test_gpu_ulysses_ranks.py.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import inputs as wl
from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp, ulysses_attn_jvp_bwd
from oracle import attn_jvp_oracle as orc

pytestmark = pytest.mark.gpu


def _close(got, ref, tol):
    g = got.double().cpu().numpy()
    err = np.abs(g - ref) / (1.0 + np.abs(ref))
    assert np.isfinite(g).all()
    assert err.max() <= tol, f"max scaled error {err.max():.3e} > {tol}"


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def nccl_group(cuda_device):
    torch.cuda.set_device(cuda_device)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0,
                            world_size=1, timeout=datetime.timedelta(seconds=60))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("d", [64, 128])
def test_ulysses_single_rank_equals_direct_call(cuda_device, nccl_group, d):
    w = wl.Workload("ulysses", B=1, H=4, d=d, n_chunks=3, chunk_tokens=150,
                    mode=wl.TEACHER_FORCING, seed=515)
    x = wl.make_inputs(w, device=cuda_device)
    ins = [x[n] for n in wl.TENSOR_ORDER]
    a = aj.attn_jvp(*ins, w.mode, w.chunk_tokens, w.n_chunks)
    b = ulysses_attn_jvp(*ins, (w.mode, w.chunk_tokens, w.n_chunks))
    torch.cuda.synchronize()
    assert aj.sync_status() == 0
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.uint8), v.contiguous().view(torch.uint8))
    O, tO, LSE = orc.attn_jvp_dense(*(t.cpu() for t in ins), w.mode, w.chunk_tokens, w.n_chunks)
    for got, ref, tol in zip(b, (O, tO, LSE), (2e-2, 2e-2, 1e-3)):
        _close(got, ref, tol)


@pytest.mark.parametrize("d", [64, 128])
def test_ulysses_backward_single_rank_equals_direct_call(cuda_device, nccl_group, d):
    w = wl.Workload("ulysses_bwd", B=1, H=4, d=d, n_chunks=3, chunk_tokens=150,
                    mode=wl.BLOCK_CAUSAL, seed=516)
    x = wl.make_inputs(w, device=cuda_device)
    q, k, v = x["q"], x["k"], x["v"]
    m = (w.mode, w.chunk_tokens, w.n_chunks)
    o, _, lse = aj.attn_jvp(q, k, v, x["tq"], x["tk"], x["tv"], *m)
    g = torch.Generator(device=cuda_device).manual_seed(7)
    do = torch.randn(q.shape, generator=g, device=cuda_device).to(q.dtype)
    a = aj.attn_jvp_bwd(q, k, v, o, do, lse, *m)
    b = ulysses_attn_jvp_bwd(q, k, v, o, do, lse, m)
    torch.cuda.synchronize()
    assert aj.sync_status() == 0
    for u, v2 in zip(a, b):
        assert torch.equal(u.view(torch.uint8), v2.contiguous().view(torch.uint8))
    ref = orc.attn_vjp_dense(q.cpu(), k.cpu(), v.cpu(), do.cpu(), *m)
    for got, r in zip(b, ref):
        _close(got, r, 2e-2)
