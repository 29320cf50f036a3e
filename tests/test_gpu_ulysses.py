"""The Ulysses path on a GPU with the library's kernel as the local attention
(NCCL process group of one rank: the exchange is the identity, the kernel and
the layout code are the real ones). Its outputs must equal a direct call's.
"""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import inputs as wl
from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp

pytestmark = pytest.mark.gpu


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
