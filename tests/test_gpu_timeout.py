"""Failure detection on the GPU without a fault: the bounded waits of the bf16
forward kernels run out, the kernel reports it, and the device stays usable.

Every wait in the kernels is bounded. A test-only setting
(attn_jvp_debug_wait) makes the first work unit's MMA issuer wait, at a
chosen key tile, on a barrier that nothing completes, with a limit of a few
milliseconds. The wait runs out; the kernel drains the copies and MMAs in
flight, frees its tensor memory and returns, and attn_jvp_sync_status must
report ATTN_JVP_ERR_DEVICE_TIMEOUT. A normal call right after, on the same
device, must match the oracle. Both kernel forms run: single CTAs (head dim
64) and CTA pairs (head dim 128, whose copies complete on the leader's
barriers, drained through the count exchange at the end of the kernel). So
does the allocation-free entry point, which reports the timeout itself and
must clear its scratch word on the next call.
"""
import ctypes

import numpy as np
import pytest
import torch

import attention_jvp_attn_b200 as aj
from attention_jvp_attn_b200 import _abi
from attention_jvp_attn_b200 import inputs as wl
from oracle import attn_jvp_oracle as orc

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture
def lib(cuda_device):
    from attention_jvp_attn_b200 import build
    build.build()
    lib = _abi.load()
    yield lib
    assert lib.attn_jvp_debug_wait(0, -1) == _abi.OK  # normal operation for later tests


def _close(got, ref, tol):
    g = got.double().cpu().numpy()
    err = np.abs(g - ref) / (1.0 + np.abs(ref))
    assert np.isfinite(g).all() and err.max() <= tol, err.max()


def _workload(d):
    return wl.Workload(f"timeout_d{d}", B=1, H=2, d=d, n_chunks=3, chunk_tokens=150,
                       mode=wl.TEACHER_FORCING, seed=900 + d)


@pytest.mark.parametrize("d,stall_tile", [(64, 0), (64, 2), (128, 0), (128, 2)])
def test_wait_runs_out_is_reported_and_the_device_stays_usable(lib, cuda_device, d, stall_tile):
    w = _workload(d)
    x = wl.make_inputs(w, device=cuda_device)
    ins = [x[n] for n in wl.TENSOR_ORDER]
    assert aj.sync_status() == 0
    assert lib.attn_jvp_debug_wait(LIMIT_NS, stall_tile) == _abi.OK
    aj.attn_jvp(*ins, w.mode, w.chunk_tokens, w.n_chunks)
    assert aj.sync_status() == _abi.ERR_DEVICE_TIMEOUT
    assert lib.attn_jvp_debug_wait(0, -1) == _abi.OK
    o, to, lse = aj.attn_jvp(*ins, w.mode, w.chunk_tokens, w.n_chunks)
    assert aj.sync_status() == 0
    O, tO, LSE = orc.attn_jvp_dense(*(t.cpu() for t in ins), w.mode, w.chunk_tokens, w.n_chunks)
    _close(o, O, 2e-2)
    _close(to, tO, 2e-2)
    _close(lse, LSE, 1e-3)


def test_noalloc_reports_the_timeout_and_clears_its_word(lib, cuda_device):
    w = _workload(128)
    x = wl.make_inputs(w, device=cuda_device)
    names = wl.TENSOR_ORDER
    ref = aj.attn_jvp(*(x[n] for n in names), w.mode, w.chunk_tokens, w.n_chunks)
    assert aj.sync_status() == 0
    shape = _abi.Shape(w.B, w.L, w.H, w.d, _abi.DTYPE_BF16, 0.0)
    mask = _abi.Mask(w.mode, w.chunk_tokens, w.n_chunks)
    stream = torch.cuda.current_stream(cuda_device).cuda_stream
    outs = [torch.empty_like(x["q"]), torch.empty_like(x["q"]),
            torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=cuda_device)]
    args = [ctypes.byref(shape), *(x[n].data_ptr() for n in names), mask,
            *(t.data_ptr() for t in outs), stream]
    assert lib.attn_jvp_debug_wait(LIMIT_NS, 1) == _abi.OK
    assert lib.attn_jvp_fwd_noalloc(*args) == _abi.ERR_DEVICE_TIMEOUT
    assert lib.attn_jvp_debug_wait(0, -1) == _abi.OK
    # the word still holds the timeout bit: the next call must clear it first
    assert lib.attn_jvp_fwd_noalloc(*args) == _abi.OK
    for got, r in zip(outs, ref):
        assert torch.equal(got.view(torch.uint8), r.view(torch.uint8))
