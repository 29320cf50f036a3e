"""Tangent-aware Ulysses context parallelism around the fused attention JVP.

Causal-rCM summary page, "Context parallelism" and "JVP and distributed
attention": the flattened token sequence is sharded across G ranks; an
all-to-all turns the sequence shards of Q, K, V into full-sequence shards of
H/G heads for local attention, and another all-to-all returns the outputs to
sequence shards. The tangents tQ, tK, tV travel with the same pattern, and so
does the tangent output tO.

Per rank, inputs are the rank's sequence block: [B, L/G, H, d] with rows
[r L/G, (r+1) L/G) of the packed sequence (r = rank in `group`). Outputs are
O and tO in the same layout and LSE as [B, H, L/G]. H and L must be multiples
of G. The mask is the full-sequence mask (every rank sees every key of its
heads after the exchange).

Communication: one all-to-all for the six inputs (stacked into one buffer),
one for O and tO, one for LSE, on the process group's backend (NCCL over
NVLink between GPUs; gloo in the CPU tests). The attention itself is the
library's kernel; `attn` can be replaced (the tests put the float64 oracle
there to check the data movement exactly).

The backward (ulysses_attn_jvp_bwd) is the transposed exchange: Q, K, V, O,
dO and LSE go to head shards, the library's backward runs on the shard, and
dQ, dK, dV go back to sequence blocks (`bwd` can be replaced likewise).
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence, Tuple

import torch
import torch.distributed as dist

from . import inputs as _wl

Tensor = torch.Tensor


def _seq_to_heads(x: Tensor, G: int, group) -> Tensor:
    """[n, B, Ls, H, d] sequence blocks -> [n, B, G*Ls, H/G, d] head blocks."""
    n, B, Ls, H, d = x.shape
    Hg = H // G
    # chunk for destination rank j: heads [j Hg, (j+1) Hg)
    send = x.reshape(n, B, Ls, G, Hg, d).permute(3, 0, 1, 2, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[s] is sequence block s of my heads
    return recv.permute(1, 2, 0, 3, 4, 5).reshape(n, B, G * Ls, Hg, d)


def _heads_to_seq(y: Tensor, G: int, group) -> Tensor:
    """[n, B, L, H/G, d] head blocks -> [n, B, L/G, H, d] sequence blocks."""
    n, B, L, Hg, d = y.shape
    Ls = L // G
    # chunk for destination rank j: sequence block j
    send = y.reshape(n, B, G, Ls, Hg, d).permute(2, 0, 1, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[s] holds heads [s Hg, (s+1) Hg) of my sequence block
    return recv.permute(1, 2, 3, 0, 4, 5).reshape(n, B, Ls, G * Hg, d)


def _lse_to_seq(lse: Tensor, G: int, group) -> Tensor:
    """[B, H/G, L] -> [B, H, L/G]."""
    B, Hg, L = lse.shape
    Ls = L // G
    send = lse.reshape(B, Hg, G, Ls).permute(2, 0, 1, 3).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3).reshape(B, G * Hg, Ls)


def _lse_to_heads(lse: Tensor, G: int, group) -> Tensor:
    """[B, H, L/G] -> [B, H/G, L] (the inverse of _lse_to_seq)."""
    B, H, Ls = lse.shape
    Hg = H // G
    # chunk for destination rank j: heads [j Hg, (j+1) Hg)
    send = lse.reshape(B, G, Hg, Ls).permute(1, 0, 2, 3).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[s] is sequence block s of my heads
    return recv.permute(1, 2, 0, 3).reshape(B, Hg, G * Ls)


def _kernel_attn(mask):
    from . import attn_jvp, attn_jvp_groups

    def run(q, k, v, tq, tk, tv, scale):
        if isinstance(mask, dict):
            return attn_jvp_groups(q, k, v, tq, tk, tv, mask["groups"], scale)
        mode, c, n = mask
        return attn_jvp(q, k, v, tq, tk, tv, mode, c, n, scale)

    return run


def ulysses_attn_jvp(q: Tensor, k: Tensor, v: Tensor, tq: Tensor, tk: Tensor, tv: Tensor,
                     mask, scale: Optional[float] = None, group=None,
                     attn: Optional[Callable[..., Tuple[Tensor, Tensor, Tensor]]] = None
                     ) -> Tuple[Tensor, Tensor, Tensor]:
    """O, tO ([B, L/G, H, d]) and LSE ([B, H, L/G]) of this rank's sequence
    block, computed by head-parallel attention over the full sequence.

    `mask` is (mode, chunk_tokens, n_chunks) or {"groups": table} for the full
    sequence; `group` a torch.distributed process group (default: world)."""
    G = dist.get_world_size(group)
    B, Ls, H, d = q.shape
    for t in (k, v, tq, tk, tv):
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, tq, tk, tv must share shape, dtype and device")
    if H % G:
        raise ValueError(f"heads ({H}) must be a multiple of the group size ({G})")
    L = Ls * G
    if isinstance(mask, dict):
        if int(mask["groups"][-1][0]) != L:
            raise ValueError("the group table does not cover the gathered sequence")
    else:
        mode, c, n = mask
        if (2 if mode == _wl.TEACHER_FORCING else 1) * n * c != L:
            raise ValueError("the mask's sequence length differs from G x the local block")
    run = attn if attn is not None else _kernel_attn(mask)
    full = _seq_to_heads(torch.stack((q, k, v, tq, tk, tv)), G, group)
    qh, kh, vh, tqh, tkh, tvh = (t.contiguous() for t in full.unbind(0))
    o, to, lse = run(qh, kh, vh, tqh, tkh, tvh, scale)
    out = _heads_to_seq(torch.stack((o, to)), G, group)
    return out[0], out[1], _lse_to_seq(lse.contiguous(), G, group)


def _kernel_bwd(mask):
    from . import attn_jvp_bwd, attn_jvp_bwd_groups

    def run(q, k, v, o, do, lse, scale, dlse):
        if isinstance(mask, dict):
            return attn_jvp_bwd_groups(q, k, v, o, do, lse, mask["groups"], scale, dlse=dlse)
        mode, c, n = mask
        return attn_jvp_bwd(q, k, v, o, do, lse, mode, c, n, scale, dlse=dlse)

    return run


def ulysses_attn_jvp_bwd(q: Tensor, k: Tensor, v: Tensor, o: Tensor, do: Tensor, lse: Tensor,
                         mask, scale: Optional[float] = None, dlse: Optional[Tensor] = None,
                         group=None, bwd: Optional[Callable[..., Tuple[Tensor, Tensor, Tensor]]] = None
                         ) -> Tuple[Tensor, Tensor, Tensor]:
    """dQ, dK, dV ([B, L/G, H, d]) of this rank's sequence block, for the
    attention that ulysses_attn_jvp computed: the transposed exchange of the
    forward. q, k, v, o, do are this rank's sequence blocks; lse (and dlse, if
    given) are [B, H, L/G] as ulysses_attn_jvp returns them. One all-to-all
    takes the five tensors to head shards over the full sequence, one takes
    LSE (and one dLSE); the backward runs on the head shard, and one
    all-to-all returns dQ, dK, dV to sequence blocks. Ulysses has no partial
    sums: every gradient row is computed whole on one rank."""
    G = dist.get_world_size(group)
    B, Ls, H, d = q.shape
    for t in (k, v, o, do):
        if t.shape != q.shape or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, o, do must share shape, dtype and device")
    if H % G:
        raise ValueError(f"heads ({H}) must be a multiple of the group size ({G})")
    for t in (lse,) + ((dlse,) if dlse is not None else ()):
        if t.shape != (B, H, Ls):
            raise ValueError("lse and dlse must be [B, H, L/G]")
    L = Ls * G
    if isinstance(mask, dict):
        if int(mask["groups"][-1][0]) != L:
            raise ValueError("the group table does not cover the gathered sequence")
    else:
        mode, c, n = mask
        if (2 if mode == _wl.TEACHER_FORCING else 1) * n * c != L:
            raise ValueError("the mask's sequence length differs from G x the local block")
    run = bwd if bwd is not None else _kernel_bwd(mask)
    full = _seq_to_heads(torch.stack((q, k, v, o, do)), G, group)
    qh, kh, vh, oh, doh = (t.contiguous() for t in full.unbind(0))
    lse_h = _lse_to_heads(lse.contiguous(), G, group).contiguous()
    dlse_h = _lse_to_heads(dlse.contiguous(), G, group).contiguous() if dlse is not None else None
    dq, dk, dv = run(qh, kh, vh, oh, doh, lse_h, scale, dlse_h)
    out = _heads_to_seq(torch.stack((dq, dk, dv)), G, group)
    return out[0], out[1], out[2]
