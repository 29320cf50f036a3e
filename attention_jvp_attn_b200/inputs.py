"""Seeded synthetic inputs for masked attention + JVP workloads.

This module only draws random tensors and describes workload shapes. It holds
none of the attention arithmetic, so both the float64 oracle (tests) and the
CUDA path (library, bench) can take their inputs from it.

Workloads follow the Causal-rCM setting (Causal-rCM summary page, App. B and
section 3 "Continuous-time consistency"): a packed sequence of clean context
chunks followed by noisy target chunks, Wan2.1-sized latent frames of 1560
tokens, frame-wise (one frame per chunk) and chunk-wise (three frames per
chunk) variants, and a plain block-causal variant without the clean/noisy
doubling. The pages give no tensors, so every value here is synthetic.

Layout of every tensor: [B, L, H, d], d innermost, contiguous.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional

import torch

TEACHER_FORCING = 0
BLOCK_CAUSAL = 1

MODE_NAMES = {TEACHER_FORCING: "teacher_forcing", BLOCK_CAUSAL: "block_causal"}

TENSOR_ORDER = ("q", "k", "v", "tq", "tk", "tv")


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention+JVP problem: shapes, mask and input distribution."""

    name: str
    B: int
    H: int
    d: int
    n_chunks: int
    chunk_tokens: int
    mode: int = TEACHER_FORCING
    dtype: str = "bf16"  # "bf16" or "f32"
    # standard deviations of the six normal draws, in TENSOR_ORDER
    stds: tuple = (1.0, 1.0, 1.0, 1.0, 1.0, 1.0)
    seed: int = 0
    scale: Optional[float] = None  # None -> 1/sqrt(d)

    @property
    def L(self) -> int:
        per = 2 if self.mode == TEACHER_FORCING else 1
        return per * self.n_chunks * self.chunk_tokens

    @property
    def softmax_scale(self) -> float:
        return self.scale if self.scale is not None else 1.0 / math.sqrt(self.d)

    def input_bytes(self) -> int:
        esz = 2 if self.dtype == "bf16" else 4
        return 6 * self.B * self.L * self.H * self.d * esz

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


_R2 = 1.0 / math.sqrt(2.0)

TINY_F32 = Workload("tiny_f32_tf", B=1, H=2, d=64, n_chunks=4, chunk_tokens=16,
                    dtype="f32", seed=1001)
FRAMEWISE_TF = Workload("framewise_tf_bf16", B=1, H=12, d=128, n_chunks=21,
                        chunk_tokens=1560, stds=(_R2, _R2, 1.0, 1.0, 1.0, 1.0),
                        seed=1002)
# "same distributions as" the frame-wise workload (its chunk-wise sibling)
CHUNKWISE_TF = Workload("chunkwise_tf_bf16", B=1, H=12, d=128, n_chunks=7,
                        chunk_tokens=4680, stds=(_R2, _R2, 1.0, 1.0, 1.0, 1.0),
                        seed=1003)
BLOCK_CAUSAL_BF16 = Workload("block_causal_bf16", B=4, H=12, d=128, n_chunks=9,
                             chunk_tokens=1560, mode=BLOCK_CAUSAL,
                             stds=(_R2, _R2, 1.0, 0.1, 0.1, 0.1), seed=1004)


def sweep_points() -> List[Workload]:
    """Teacher-forcing sweep: H=16, d in {64,128}, chunk sizes 256/1560/4680,
    sequences 4k-128k tokens, batch filling at most 8 GiB of bf16 inputs."""
    n_for_c = {256: (8, 32, 64, 128, 256), 1560: (2, 6, 11, 21, 42),
               4680: (1, 2, 4, 7, 14)}
    pts = []
    idx = 0
    for d in (64, 128):
        for c, ns in n_for_c.items():
            for n in ns:
                L = 2 * n * c
                B = max(1, (8 << 30) // (12 * L * 16 * d))
                pts.append(Workload(f"sweep_d{d}_c{c}_n{n}", B=B, H=16, d=d,
                                    n_chunks=n, chunk_tokens=c, seed=5000 + idx))
                idx += 1
    return pts


WORKLOADS: Dict[str, Workload] = {w.name: w for w in
                                  (TINY_F32, FRAMEWISE_TF, CHUNKWISE_TF, BLOCK_CAUSAL_BF16)}
for _w in sweep_points():
    WORKLOADS[_w.name] = _w


def make_inputs(w: Workload, device="cpu", seed: Optional[int] = None,
                batch: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw q, k, v, tq, tk, tv (in that order) from one seeded generator on
    `device`, in fp32, scale each by its std and cast (round to nearest even)
    to the workload dtype. `batch` overrides B (used for bounded samples)."""
    B = w.B if batch is None else batch
    g = torch.Generator(device=device)
    g.manual_seed(w.seed if seed is None else seed)
    shape = (B, w.L, w.H, w.d)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    out = {}
    for name, std in zip(TENSOR_ORDER, w.stds):
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        out[name] = x.to(dt)
        del x
    return out


def sample_rows(w: Workload, n_random: int = 256, seed: int = 7,
                tile: int = 128, max_rows: Optional[int] = None) -> List[int]:
    """Query rows worth checking one by one on a large workload: first and
    last row of every chunk (clean and noisy), the rows on both sides of the
    `tile` boundaries around every chunk boundary (where tiles are partial),
    the ragged tail, and `n_random` seeded random rows. With `max_rows`, a
    seeded subset of that size (always keeping the first and last row)."""
    L, c = w.L, w.chunk_tokens
    rows = set()
    for j in range(L // c):
        p = j * c
        rows.update((p, p + c - 1))
        t = p // tile
        for q in (t * tile - 1, t * tile, (t + 1) * tile - 1, (t + 1) * tile):
            rows.add(q)
    rows.update((L - 1, (L - 1) // tile * tile, (L - 1) // tile * tile - 1))
    g = torch.Generator().manual_seed(seed)
    rows.update(torch.randint(0, L, (n_random,), generator=g).tolist())
    out = sorted(r for r in rows if 0 <= r < L)
    if max_rows is not None and len(out) > max_rows:
        keep = torch.randperm(len(out), generator=g)[:max_rows - 2].tolist()
        out = sorted({out[0], out[-1], *(out[i] for i in keep)})
    return out
