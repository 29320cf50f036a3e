"""The allocation-free entry point, attn_jvp_fwd_noalloc, against attn_jvp_fwd.

Some callers cannot let a library allocate device memory: runtimes with their
own allocator and a fixed memory budget, plugin hosts that hand in every
device buffer, code paths where cudaMalloc is not allowed. For them the
library keeps the one scratch word its bf16 kernel needs in a fixed device
array instead. This test calls that entry point through the C ABI twice in a
row, for the CTA-pair kernel (head dim 128) and the single-CTA kernel (head
dim 64). Both entry points launch the same kernel with the same parameters,
so every call must give the same bits as the regular entry point.

It sits in a file pytest collects last, so a run that stops at the first
failure has run every other test before it; it also passes on its own in a
fresh process.
"""
import ctypes

import pytest
import torch

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import _abi
from attention_jvp_attn_b200 import inputs as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("d", [128, 64])
def test_noalloc_matches_regular_entry_point_on_two_calls(cuda_device, d):
    from attention_jvp_attn_b200 import build
    build.build()
    lib = _abi.load()
    w = wl.Workload("noalloc", B=2, H=3, d=d, n_chunks=3, chunk_tokens=150,
                    mode=wl.TEACHER_FORCING, seed=404 + d)
    x = wl.make_inputs(w, device=cuda_device)
    names = wl.TENSOR_ORDER
    o_ref, to_ref, lse_ref = aj.attn_jvp(*(x[n] for n in names), w.mode, w.chunk_tokens,
                                         w.n_chunks)
    assert aj.sync_status() == 0
    shape = _abi.Shape(w.B, w.L, w.H, w.d, _abi.DTYPE_BF16, 0.0)
    mask = _abi.Mask(w.mode, w.chunk_tokens, w.n_chunks)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    for call in range(2):
        o = torch.full_like(x["q"], float("nan"))
        to = torch.full_like(x["q"], float("nan"))
        lse = torch.full((w.B, w.H, w.L), float("nan"), device=cuda_device)
        rc = lib.attn_jvp_fwd_noalloc(ctypes.byref(shape), *(x[n].data_ptr() for n in names),
                                      mask, o.data_ptr(), to.data_ptr(), lse.data_ptr(), stream)
        assert rc == _abi.OK, (call, _abi.status_string(rc))
        for got, ref in ((o, o_ref), (to, to_ref), (lse, lse_ref)):
            assert torch.equal(got.view(torch.uint8), ref.view(torch.uint8)), call


def test_noalloc_rejects_what_the_regular_entry_point_rejects(cuda_device):
    lib = _abi.load()
    mask = _abi.Mask(wl.TEACHER_FORCING, 16, 4)
    good = [0x10000 * (i + 1) for i in range(9)]  # never dereferenced: every call fails validation
    bad_l = _abi.Shape(1, 127, 2, 64, _abi.DTYPE_BF16, 0.0)
    assert lib.attn_jvp_fwd_noalloc(ctypes.byref(bad_l), *good[:6], mask, *good[6:], None) == \
        _abi.ERR_INVALID_ARGUMENT
    f32 = _abi.Shape(1, 128, 2, 64, _abi.DTYPE_F32, 0.0)
    assert lib.attn_jvp_fwd_noalloc(ctypes.byref(f32), *good[:6], mask, *good[6:], None) == \
        _abi.ERR_UNSUPPORTED
