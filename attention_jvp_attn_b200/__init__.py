"""Custom-mask attention forward fused with its JVP, for NVIDIA B200 (sm_100a).

Given Q, K, V and tangents tQ, tK, tV ([B, L, H, d] CUDA tensors), returns
O = softmax(s Q K^T + M) V, tO = tP V + P tV with tP = P * (tS - rowsum(P * tS)),
tS = s (tQ K^T + Q tK^T), and LSE = log sum exp(s Q K^T + M) ([B, H, L] fp32),
for the teacher-forcing mask over a [clean chunks | noisy chunks] sequence or a
block-causal mask (Causal-rCM summary page, App. B). All arithmetic runs in the
CUDA library behind the C ABI (include/attn_jvp.h); this module only checks
tensors and passes pointers and the current stream.
"""
from __future__ import annotations

import ctypes
import math
from typing import List, Optional, Sequence, Tuple

import torch

from . import _abi
from ._abi import AttnJvpError  # noqa: F401
from .inputs import BLOCK_CAUSAL, TEACHER_FORCING  # noqa: F401

__all__ = ["attn_jvp", "attn_jvp_groups", "attn_jvp_bwd", "attn_jvp_bwd_groups", "rope",
           "attn_jvp_rope", "attn_jvp_host", "sync_status", "unmasked_pairs", "schedule_tiles",
           "key_tile_query_bounds", "host_staging_bytes", "AttnJvpError", "TEACHER_FORCING",
           "BLOCK_CAUSAL"]

_DT = {torch.bfloat16: _abi.DTYPE_BF16, torch.float32: _abi.DTYPE_F32}


def _shape(q: torch.Tensor, scale: Optional[float]) -> _abi.Shape:
    if q.dim() != 4:
        raise ValueError("expected [B, L, H, d] tensors")
    if q.dtype not in _DT:
        raise TypeError(f"unsupported dtype {q.dtype} (bf16 or fp32)")
    B, L, H, d = q.shape
    return _abi.Shape(B, L, H, d, _DT[q.dtype], float(scale) if scale is not None else 0.0)


def _mask(mode: int, chunk_tokens: int, n_chunks: int) -> _abi.Mask:
    return _abi.Mask(int(mode), int(chunk_tokens), int(n_chunks))


def _stream_handle(device: torch.device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def attn_jvp(q, k, v, tq, tk, tv, mode: int, chunk_tokens: int, n_chunks: int,
             scale: Optional[float] = None,
             out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None):
    """O, tO ([B, L, H, d], input dtype) and LSE ([B, H, L], fp32) on the
    current CUDA stream. `scale` defaults to 1/sqrt(d)."""
    ts = (q, k, v, tq, tk, tv)
    for t in ts:
        if not t.is_cuda:
            raise ValueError("inputs must be CUDA tensors")
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, tq, tk, tv must share shape, dtype and device")
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous [B, L, H, d]")
    shape = _shape(q, scale)
    B, L, H, d = q.shape
    if out is None:
        o = torch.empty_like(q)
        to = torch.empty_like(q)
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    else:
        o, to, lse = out
    lib = _abi.load()
    with torch.cuda.device(q.device):
        rc = lib.attn_jvp_fwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                              tq.data_ptr(), tk.data_ptr(), tv.data_ptr(),
                              _mask(mode, chunk_tokens, n_chunks),
                              o.data_ptr(), to.data_ptr(), lse.data_ptr(),
                              _stream_handle(q.device))
    _abi.check(rc, "attn_jvp_fwd")
    return o, to, lse


def attn_jvp_groups(q, k, v, tq, tk, tv, groups: Sequence[Tuple[int, int, int, int, int]],
                    scale: Optional[float] = None,
                    out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None):
    """attn_jvp with a general mask: `groups` is a table of
    (row_end, k0_begin, k0_end, k1_begin, k1_end) row groups in row order, the
    last ending at L; rows of a group may attend to keys [k0_begin, k0_end)
    and [k1_begin, k1_end)."""
    ts = (q, k, v, tq, tk, tv)
    for t in ts:
        if not t.is_cuda:
            raise ValueError("inputs must be CUDA tensors")
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, tq, tk, tv must share shape, dtype and device")
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous [B, L, H, d]")
    shape = _shape(q, scale)
    B, L, H, d = q.shape
    if out is None:
        o = torch.empty_like(q)
        to = torch.empty_like(q)
        lse = torch.empty((B, H, L), dtype=torch.float32, device=q.device)
    else:
        o, to, lse = out
    table = _abi.group_array(groups)
    lib = _abi.load()
    with torch.cuda.device(q.device):
        rc = lib.attn_jvp_fwd_groups(ctypes.byref(shape), q.data_ptr(), k.data_ptr(),
                                     v.data_ptr(), tq.data_ptr(), tk.data_ptr(), tv.data_ptr(),
                                     table, len(groups), o.data_ptr(), to.data_ptr(),
                                     lse.data_ptr(), _stream_handle(q.device))
    _abi.check(rc, "attn_jvp_fwd_groups")
    return o, to, lse


def _bwd_args(q, k, v, o, do, lse, dlse, scale, out):
    for t in (q, k, v, o, do):
        if not t.is_cuda:
            raise ValueError("inputs must be CUDA tensors")
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, o, do must share shape, dtype and device")
        if not t.is_contiguous():
            raise ValueError("inputs must be contiguous [B, L, H, d]")
    B, L, H, d = q.shape
    for t in (lse,) + ((dlse,) if dlse is not None else ()):
        if t.shape != (B, H, L) or t.dtype != torch.float32 or t.device != q.device \
                or not t.is_contiguous():
            raise ValueError("lse and dlse must be contiguous fp32 [B, H, L] on the inputs' device")
    shape = _shape(q, scale)
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(q), torch.empty_like(q))
    return shape, out


def attn_jvp_bwd(q, k, v, o, do, lse, mode: int, chunk_tokens: int, n_chunks: int,
                 scale: Optional[float] = None, dlse: Optional[torch.Tensor] = None,
                 out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None):
    """dQ, dK, dV ([B, L, H, d], input dtype) of the masked primal attention,
    from the forward's inputs, its output O and LSE, the cotangent dO of O and
    optionally a cotangent dLSE of LSE ([B, H, L] fp32), on the current stream."""
    shape, (dq, dk, dv) = _bwd_args(q, k, v, o, do, lse, dlse, scale, out)
    lib = _abi.load()
    with torch.cuda.device(q.device):
        rc = lib.attn_jvp_bwd(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), v.data_ptr(),
                              o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                              dlse.data_ptr() if dlse is not None else None,
                              _mask(mode, chunk_tokens, n_chunks),
                              dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                              _stream_handle(q.device))
    _abi.check(rc, "attn_jvp_bwd")
    return dq, dk, dv


def attn_jvp_bwd_groups(q, k, v, o, do, lse, groups: Sequence[Tuple[int, int, int, int, int]],
                        scale: Optional[float] = None, dlse: Optional[torch.Tensor] = None,
                        out: Optional[Tuple[torch.Tensor, torch.Tensor, torch.Tensor]] = None):
    """attn_jvp_bwd with a group-table mask (as for attn_jvp_groups)."""
    shape, (dq, dk, dv) = _bwd_args(q, k, v, o, do, lse, dlse, scale, out)
    table = _abi.group_array(groups)
    lib = _abi.load()
    with torch.cuda.device(q.device):
        rc = lib.attn_jvp_bwd_groups(ctypes.byref(shape), q.data_ptr(), k.data_ptr(),
                                     v.data_ptr(), o.data_ptr(), do.data_ptr(), lse.data_ptr(),
                                     dlse.data_ptr() if dlse is not None else None,
                                     table, len(groups), dq.data_ptr(), dk.data_ptr(),
                                     dv.data_ptr(), _stream_handle(q.device))
    _abi.check(rc, "attn_jvp_bwd_groups")
    return dq, dk, dv


def rope(q, k, tq, tk, cos, sin, out=None):
    """Rotary position embedding of q, k and their tangents tq, tk
    ([B, L, H, d] CUDA tensors) by per-token angles: cos, sin are fp32 [L, d/2]
    tables. Returns the four rotated tensors (`out` may be the inputs
    themselves, for an in-place rotation)."""
    for t in (q, k, tq, tk):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, tq, tk must share shape, dtype and device")
    B, L, H, d = q.shape
    for t in (cos, sin):
        if t.shape != (L, d // 2) or t.dtype != torch.float32 or t.device != q.device \
                or not t.is_contiguous():
            raise ValueError("cos and sin must be contiguous fp32 [L, d/2] on the inputs' device")
    shape = _shape(q, None)
    if out is None:
        out = tuple(torch.empty_like(q) for _ in range(4))
    lib = _abi.load()
    with torch.cuda.device(q.device):
        rc = lib.attn_jvp_rope(ctypes.byref(shape), q.data_ptr(), k.data_ptr(), tq.data_ptr(),
                               tk.data_ptr(), cos.data_ptr(), sin.data_ptr(),
                               *(t.data_ptr() for t in out), _stream_handle(q.device))
    _abi.check(rc, "attn_jvp_rope")
    return out


def attn_jvp_rope(q, k, v, tq, tk, tv, cos, sin, mode: int, chunk_tokens: int, n_chunks: int,
                  scale: Optional[float] = None, return_rotated: bool = False, out=None,
                  rotated=None):
    """The attention JVP with RoPE applied to the queries and keys (and their
    tangents) first, in one call (one kernel launch for bf16): returns
    (o, to, lse), and also the rotated (q, k, tq, tk) with return_rotated.
    `rotated` may give the four buffers for the rotated tensors (the inputs
    themselves for an in-place rotation)."""
    ts = (q, k, v, tq, tk, tv)
    for t in ts:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous CUDA tensors")
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, tq, tk, tv must share shape, dtype and device")
    B, L, H, d = q.shape
    for t in (cos, sin):
        if t.shape != (L, d // 2) or t.dtype != torch.float32 or t.device != q.device \
                or not t.is_contiguous():
            raise ValueError("cos and sin must be contiguous fp32 [L, d/2] on the inputs' device")
    shape = _shape(q, scale)
    rot = rotated if rotated is not None else tuple(torch.empty_like(q) for _ in range(4))
    if out is None:
        out = (torch.empty_like(q), torch.empty_like(q),
               torch.empty((B, H, L), dtype=torch.float32, device=q.device))
    lib = _abi.load()
    with torch.cuda.device(q.device):
        rc = lib.attn_jvp_fwd_rope(ctypes.byref(shape), *(t.data_ptr() for t in ts),
                                   cos.data_ptr(), sin.data_ptr(),
                                   _mask(mode, chunk_tokens, n_chunks),
                                   *(t.data_ptr() for t in rot), *(t.data_ptr() for t in out),
                                   _stream_handle(q.device))
    _abi.check(rc, "attn_jvp_fwd_rope")
    return (tuple(out), tuple(rot)) if return_rotated else tuple(out)


def host_staging_bytes(B: int, L: int, H: int, d: int, dtype: torch.dtype) -> int:
    shape = _abi.Shape(B, L, H, d, _DT[dtype], 0.0)
    return int(_abi.load().attn_jvp_host_staging_bytes(ctypes.byref(shape)))


def attn_jvp_host(q, k, v, tq, tk, tv, mode: int, chunk_tokens: int, n_chunks: int,
                  staging: torch.Tensor, out, scale: Optional[float] = None,
                  device: Optional[torch.device] = None) -> None:
    """Same operation on HOST tensors (pinned for full copy speed): copies the
    inputs in, runs, copies O, tO, LSE back into `out` and waits. `staging` is
    a uint8 CUDA tensor of at least host_staging_bytes(...) bytes."""
    o, to, lse = out
    for t in (q, k, v, tq, tk, tv, o, to, lse):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host path takes contiguous CPU tensors")
    shape = _shape(q, scale)
    dev = staging.device if device is None else device
    lib = _abi.load()
    with torch.cuda.device(dev):
        rc = lib.attn_jvp_fwd_host(ctypes.byref(shape), q.data_ptr(), k.data_ptr(),
                                   v.data_ptr(), tq.data_ptr(), tk.data_ptr(), tv.data_ptr(),
                                   _mask(mode, chunk_tokens, n_chunks), o.data_ptr(),
                                   to.data_ptr(), lse.data_ptr(), staging.data_ptr(),
                                   _stream_handle(dev))
    _abi.check(rc, "attn_jvp_fwd_host")


def sync_status(device: Optional[torch.device] = None) -> int:
    """Synchronize the current stream and return (and clear) the library's
    device status (0 = ok, 5 = a kernel's bounded wait ran out)."""
    dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
    with torch.cuda.device(dev):
        return int(_abi.load().attn_jvp_sync_status(_stream_handle(dev)))


def unmasked_pairs(mode: int, chunk_tokens: int, n_chunks: int) -> int:
    """Admissible (query, key) pairs per (batch, head)."""
    return int(_abi.load().attn_jvp_unmasked_pairs(_mask(mode, chunk_tokens, n_chunks)))


def schedule_tiles(mode: int, chunk_tokens: int, n_chunks: int, L: int, block_m: int,
                   block_n: int, q_tile: int) -> Tuple[List[int], List[int]]:
    """Key tiles (and their full/partial flags) the kernels visit for one query tile."""
    lib = _abi.load()
    m = _mask(mode, chunk_tokens, n_chunks)
    n = lib.attn_jvp_schedule_tiles(m, L, block_m, block_n, q_tile, None, None, 0)
    if n < 0:
        raise ValueError("bad schedule arguments")
    tiles = (ctypes.c_int32 * max(n, 1))()
    full = (ctypes.c_uint8 * max(n, 1))()
    lib.attn_jvp_schedule_tiles(m, L, block_m, block_n, q_tile, tiles, full, n)
    return list(tiles[:n]), list(full[:n])


def key_tile_query_bounds(mode: int, chunk_tokens: int, n_chunks: int, L: int, block_m: int,
                          block_n: int, k_tile: int) -> Tuple[int, int]:
    """Query tiles [lo, hi] the backward scans for one key tile."""
    lo, hi = ctypes.c_int32(), ctypes.c_int32()
    r = _abi.load().attn_jvp_key_tile_query_bounds(_mask(mode, chunk_tokens, n_chunks), L, block_m,
                                                   block_n, k_tile, ctypes.byref(lo),
                                                   ctypes.byref(hi))
    if r != 0:
        raise ValueError("bad bounds arguments")
    return lo.value, hi.value


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)
