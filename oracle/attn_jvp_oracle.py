"""Float64 CPU oracle for custom-mask attention and its Jacobian-vector product.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import this module:
only tests, the smoke check and the benchmark's CPU-baseline leg use it. It
shares no code with the CUDA library.

What it computes (Causal-rCM summary page, App. B "FlashAttention-2 JVP Kernel
with Custom Masks"): for every query row i, with admissible key set A(i) given
by the mask predicate below,

    S_ij  = s * (q_i . k_j)                              j in A(i)
    LSE_i = log sum_{j in A(i)} exp(S_ij)                (natural log)
    P_ij  = exp(S_ij - LSE_i),  P_ij = 0 for j not in A(i)
    O_i   = sum_j P_ij v_j
    tS_ij = s * (tq_i . k_j + q_i . tk_j)
    mu_i  = sum_j P_ij tS_ij
    tO_i  = sum_j P_ij (tS_ij - mu_i) v_j + sum_j P_ij tv_j

This is the plain dense definition of O = softmax(S + M) V and of its
directional derivative along (tq, tk, tv): the derivative of the softmax row
is tP = P * (tS - rowsum(P * tS)), masked entries carry no tangent because the
discrete mask has none (App. B), and tO = tP V + P tV. It is evaluated
directly, not through the online-softmax recurrence the kernel uses.

Mask (App. B; section 3 "Continuous-time consistency": the TF-masked packed
forward; Causal Forcing summary page, section 2: clean and noisy videos
concatenated under a causal attention mask). The sequence is
[clean chunks | noisy chunks], n chunks of c tokens each, L = 2 n c:
  * a clean query in chunk j sees clean keys in chunks <= j and no noisy key;
  * a noisy query in chunk i sees clean keys in chunks < i and the noisy keys
    of its own chunk i.
Block-causal mode (Causal-rCM page, section 2 "Autoregressive video
diffusion": causal over temporal blocks, full attention inside a block):
L = n c and a query in chunk j sees keys in chunks <= j.
Attention inside a chunk is full (bidirectional).

General masks (App. B: the kernel takes masks as query groups with admissible
key ranges): a table of groups, each a run of consecutive query rows that
share an admissible key set made of at most two key ranges. The groups cover
the rows [0, L) in order; group g holds rows [row_end of g-1, row_end of g)
(0 for the first) and admits keys [k0_begin, k0_end) and [k1_begin, k1_end).

Backward (for training the student; the pages return LSE so that a backward
pass can rebuild P): attn_vjp_rows / attn_vjp_dense give dQ, dK, dV from an
output cotangent dO and an optional LSE cotangent, pinned separately by
tests/test_oracle_vjp_pins.py.

Rotary position embedding of queries and keys (and their tangents) before
the attention: rope_rotate / attn_jvp_rope_dense, pinned by
tests/test_oracle_rope_pins.py.

Every function here is pinned by tests/test_oracle_pins.py against values
that do not come from this file: finite differences, an autodiff JVP of the
library softmax attention, hand-derived closed forms, hand-written masks,
invariants and pair-count formulas.
"""
from __future__ import annotations

import math
from typing import Iterable, Optional, Sequence, Tuple

import numpy as np

TEACHER_FORCING = 0
BLOCK_CAUSAL = 1

# One row group: (row_end, k0_begin, k0_end, k1_begin, k1_end).
Group = Tuple[int, int, int, int, int]


def seq_len(mode: int, chunk_tokens: int, n_chunks: int) -> int:
    """L = 2 n c for the packed teacher-forcing sequence, n c otherwise."""
    return (2 if mode == TEACHER_FORCING else 1) * n_chunks * chunk_tokens


def allowed(mode: int, c: int, n: int, i, j) -> np.ndarray:
    """Mask predicate: True where query token i may attend to key token j.

    `i` and `j` broadcast against each other (0-based token indices)."""
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    if mode == BLOCK_CAUSAL:
        return (j // c) <= (i // c)
    if mode != TEACHER_FORCING:
        raise ValueError(f"unknown mask mode {mode}")
    nc = n * c
    i_clean = i < nc
    j_clean = j < nc
    ci = np.where(i_clean, i // c, (i - nc) // c)     # chunk of the query
    cj = np.where(j_clean, j // c, (j - nc) // c)     # chunk of the key
    clean_q = i_clean & j_clean & (cj <= ci)
    noisy_q_clean_k = (~i_clean) & j_clean & (cj < ci)
    noisy_q_noisy_k = (~i_clean) & (~j_clean) & (cj == ci)
    return clean_q | noisy_q_clean_k | noisy_q_noisy_k


def allowed_groups(groups: Sequence[Group], i, j) -> np.ndarray:
    """Mask predicate of a group table: True where query row i may attend to
    key j (`i` and `j` broadcast against each other)."""
    i = np.asarray(i, dtype=np.int64)
    j = np.asarray(j, dtype=np.int64)
    g = np.asarray(groups, dtype=np.int64).reshape(-1, 5)
    # the group of row i: the first whose row_end exceeds i
    gi = np.searchsorted(g[:, 0], i, side="right")
    if np.any(gi >= g.shape[0]):
        raise ValueError("row beyond the last group")
    k0b, k0e, k1b, k1e = (g[gi, c] for c in range(1, 5))
    return ((j >= k0b) & (j < k0e)) | ((j >= k1b) & (j < k1e))


def group_table(mode: int, c: int, n: int):
    """The teacher-forcing or block-causal mask written as a group table: one
    group per chunk of query rows (clean chunks, then noisy chunks)."""
    nc = n * c
    if mode == BLOCK_CAUSAL:
        return [((j + 1) * c, 0, (j + 1) * c, (j + 1) * c, (j + 1) * c) for j in range(n)]
    if mode != TEACHER_FORCING:
        raise ValueError(f"unknown mask mode {mode}")
    clean = [((j + 1) * c, 0, (j + 1) * c, (j + 1) * c, (j + 1) * c) for j in range(n)]
    noisy = [(nc + (i + 1) * c, 0, i * c, nc + i * c, nc + (i + 1) * c) for i in range(n)]
    return clean + noisy


def mask_matrix_groups(groups: Sequence[Group]) -> np.ndarray:
    """Explicit [L, L] boolean mask of a group table (small L only)."""
    L = int(groups[-1][0])
    t = np.arange(L)
    return allowed_groups(groups, t[:, None], t[None, :])


def mask_matrix(mode: int, c: int, n: int) -> np.ndarray:
    """Explicit [L, L] boolean mask (small L only)."""
    L = seq_len(mode, c, n)
    t = np.arange(L)
    return allowed(mode, c, n, t[:, None], t[None, :])


def count_pairs_bruteforce(mode: int, c: int, n: int) -> int:
    """Number of admissible (query, key) pairs, counted from the predicate."""
    L = seq_len(mode, c, n)
    t = np.arange(L)
    total = 0
    for i0 in range(0, L, 4096):
        rows = t[i0:i0 + 4096]
        total += int(allowed(mode, c, n, rows[:, None], t[None, :]).sum())
    return total


def _as64(x) -> np.ndarray:
    """Promote a tensor (numpy or torch, any float dtype) to float64 numpy,
    bit-exactly for bf16/fp32 inputs."""
    if hasattr(x, "detach"):  # torch tensor: bf16 has no numpy dtype
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def attn_jvp_rows(q, k, v, tq, tk, tv, mode: int, c: int, n: int,
                  scale: Optional[float], rows: Sequence[int],
                  block: int = 64, groups: Optional[Sequence[Group]] = None
                  ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """O, tO and LSE for the given query rows of ONE (batch, head).

    q..tv are [L, d] (any float type; promoted to float64). The mask is the
    group table `groups` if given, else (mode, c, n). Returns O [R, d],
    tO [R, d], LSE [R] in float64 for R = len(rows)."""
    q, k, v, tq, tk, tv = (_as64(x) for x in (q, k, v, tq, tk, tv))
    L, d = q.shape
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    rows = np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]
    O = np.empty((R, d))
    tO = np.empty((R, d))
    lse = np.empty(R)
    keys = np.arange(L)
    for r0 in range(0, R, block):
        rr = rows[r0:r0 + block]
        if groups is not None:
            M = allowed_groups(groups, rr[:, None], keys[None, :])    # [r, L]
        else:
            M = allowed(mode, c, n, rr[:, None], keys[None, :])       # [r, L]
        S = s * (q[rr] @ k.T)                                        # [r, L]
        S = np.where(M, S, -np.inf)
        smax = S.max(axis=1, keepdims=True)                          # finite: A(i) is never empty
        lse_r = smax[:, 0] + np.log(np.exp(S - smax).sum(axis=1))
        P = np.exp(S - lse_r[:, None])                               # 0 where masked
        tS = s * (tq[rr] @ k.T + q[rr] @ tk.T)
        tS = np.where(M, tS, 0.0)
        mu = (P * tS).sum(axis=1, keepdims=True)
        tP = P * (tS - mu)
        O[r0:r0 + block] = P @ v
        tO[r0:r0 + block] = tP @ v + P @ tv
        lse[r0:r0 + block] = lse_r
    return O, tO, lse


def attn_jvp_dense(q, k, v, tq, tk, tv, mode: int, c: int, n: int,
                   scale: Optional[float] = None,
                   groups: Optional[Sequence[Group]] = None):
    """Full outputs for [B, L, H, d] inputs: O, tO [B, L, H, d] and LSE
    [B, H, L], all float64 numpy. The mask is the group table `groups` if
    given, else (mode, c, n)."""
    q, k, v, tq, tk, tv = (_as64(x) for x in (q, k, v, tq, tk, tv))
    B, L, H, d = q.shape
    if groups is not None:
        if L != int(groups[-1][0]):
            raise ValueError("L does not match the group table")
    elif L != seq_len(mode, c, n):
        raise ValueError("L does not match the mask (mode, chunk_tokens, n_chunks)")
    O = np.empty((B, L, H, d))
    tO = np.empty((B, L, H, d))
    lse = np.empty((B, H, L))
    allrows = np.arange(L)
    for b in range(B):
        for h in range(H):
            o_, to_, l_ = attn_jvp_rows(q[b, :, h], k[b, :, h], v[b, :, h],
                                        tq[b, :, h], tk[b, :, h], tv[b, :, h],
                                        mode, c, n, scale, allrows, groups=groups)
            O[b, :, h] = o_
            tO[b, :, h] = to_
            lse[b, h] = l_
    return O, tO, lse


def attn_forward_dense(q, k, v, mode: int, c: int, n: int,
                       scale: Optional[float] = None, groups: Optional[Sequence[Group]] = None):
    """Primal output only (O and LSE); used to take finite differences and as
    the forward whose O and LSE a backward pass starts from."""
    z = np.zeros_like(_as64(q))
    O, _, lse = attn_jvp_dense(q, k, v, z, z, z, mode, c, n, scale, groups=groups)
    return O, lse


def attn_vjp_rows(q, k, v, do, mode: int, c: int, n: int, scale: Optional[float],
                  dlse=None, groups: Optional[Sequence[Group]] = None
                  ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Backward (vector-Jacobian product) of the masked primal attention of ONE
    (batch, head): given the output cotangent dO [L, d] (and optionally a
    cotangent dLSE [L] of the log-sum-exp), returns dQ, dK, dV [L, d].

    This is the gradient the primal network needs during training; the pages
    return LSE with the forward so a backward pass can rebuild P from it
    (Causal-rCM summary page, App. B, last item). Plain definition, with P the
    masked softmax of S = s q k^T:
        dV = P^T dO
        dP = dO V^T
        Delta_i = sum_j P_ij dP_ij   (= dO_i . O_i)
        dS = P * (dP - Delta) + P * dLSE_i
        dQ = s dS K,   dK = s dS^T Q
    (d LSE_i / d S_ij = P_ij gives the last term of dS.)"""
    q, k, v, do = (_as64(x) for x in (q, k, v, do))
    L, d = q.shape
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    t = np.arange(L)
    if groups is not None:
        M = allowed_groups(groups, t[:, None], t[None, :])
    else:
        M = allowed(mode, c, n, t[:, None], t[None, :])
    S = np.where(M, s * (q @ k.T), -np.inf)
    smax = S.max(axis=1, keepdims=True)
    lse = smax[:, 0] + np.log(np.exp(S - smax).sum(axis=1))
    P = np.exp(S - lse[:, None])
    dV = P.T @ do
    dP = do @ v.T
    delta = (P * dP).sum(axis=1, keepdims=True)
    dS = P * (dP - delta)
    if dlse is not None:
        dS = dS + P * _as64(dlse)[:, None]
    dQ = s * (dS @ k)
    dK = s * (dS.T @ q)
    return dQ, dK, dV


def _vjp_row_block(q, k, v, do, M, s, rr, dlse):
    """P, dP and D (= rowsum(P * dP) - dLSE) of the query rows rr over all
    keys, with M the [len(rr), L] admissible pattern."""
    S = np.where(M, s * (q[rr] @ k.T), -np.inf)
    smax = S.max(axis=1, keepdims=True)
    lse = smax[:, 0] + np.log(np.exp(S - smax).sum(axis=1))
    P = np.exp(S - lse[:, None])
    dP = do[rr] @ v.T
    D = (P * dP).sum(axis=1)
    if dlse is not None:
        D = D - dlse[rr]
    return P, dP, D


def attn_vjp_dq_rows(q, k, v, do, mode: int, c: int, n: int, scale: Optional[float],
                     rows: Sequence[int], dlse=None, groups: Optional[Sequence[Group]] = None,
                     block: int = 64) -> np.ndarray:
    """dQ [R, d] for the given query rows of ONE (batch, head): the rows of
    attn_vjp_rows' dQ, each from its own row of P (the same definition; only
    the rows asked for are formed). dlse, if given, is the [L] cotangent."""
    q, k, v, do = (_as64(x) for x in (q, k, v, do))
    dl = None if dlse is None else _as64(dlse)
    L, d = q.shape
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    rows = np.asarray(rows, dtype=np.int64)
    keys = np.arange(L)
    out = np.empty((rows.shape[0], d))
    for r0 in range(0, rows.shape[0], block):
        rr = rows[r0:r0 + block]
        M = allowed_groups(groups, rr[:, None], keys[None, :]) if groups is not None \
            else allowed(mode, c, n, rr[:, None], keys[None, :])
        P, dP, D = _vjp_row_block(q, k, v, do, M, s, rr, dl)
        out[r0:r0 + block] = s * ((P * (dP - D[:, None])) @ k)
    return out


def attn_vjp_dkdv_cols(q, k, v, do, mode: int, c: int, n: int, scale: Optional[float],
                       cols: Sequence[int], dlse=None, groups: Optional[Sequence[Group]] = None,
                       block: int = 256) -> Tuple[np.ndarray, np.ndarray]:
    """dK, dV [C, d] for the given key columns of ONE (batch, head): column j
    sums over the rows that may attend to key j, each row's P and D taken
    from that whole row (the same definition as attn_vjp_rows, only the
    columns asked for are formed). Cost grows with the number of rows that
    attend to the columns."""
    q, k, v, do = (_as64(x) for x in (q, k, v, do))
    dl = None if dlse is None else _as64(dlse)
    L, d = q.shape
    s = (1.0 / math.sqrt(d)) if scale is None else float(scale)
    cols = np.asarray(cols, dtype=np.int64)
    keys = np.arange(L)
    t = np.arange(L)
    seen = allowed_groups(groups, t[:, None], cols[None, :]) if groups is not None \
        else allowed(mode, c, n, t[:, None], cols[None, :])
    rows = np.nonzero(seen.any(axis=1))[0]
    dK = np.zeros((cols.shape[0], d))
    dV = np.zeros((cols.shape[0], d))
    for r0 in range(0, rows.shape[0], block):
        rr = rows[r0:r0 + block]
        M = allowed_groups(groups, rr[:, None], keys[None, :]) if groups is not None \
            else allowed(mode, c, n, rr[:, None], keys[None, :])
        P, dP, D = _vjp_row_block(q, k, v, do, M, s, rr, dl)
        Pc = P[:, cols]
        dSc = Pc * (dP[:, cols] - D[:, None])
        dV += Pc.T @ do[rr]
        dK += s * (dSc.T @ q[rr])
    return dK, dV


def attn_vjp_dense(q, k, v, do, mode: int, c: int, n: int, scale: Optional[float] = None,
                   dlse=None, groups: Optional[Sequence[Group]] = None):
    """dQ, dK, dV [B, L, H, d] for [B, L, H, d] inputs and output cotangent dO
    (dLSE [B, H, L] optional), all float64 numpy."""
    q, k, v, do = (_as64(x) for x in (q, k, v, do))
    B, L, H, d = q.shape
    dQ, dK, dV = (np.empty((B, L, H, d)) for _ in range(3))
    for b in range(B):
        for h in range(H):
            g = attn_vjp_rows(q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h], mode, c, n, scale,
                              None if dlse is None else _as64(dlse)[b, h], groups)
            dQ[b, :, h], dK[b, :, h], dV[b, :, h] = g
    return dQ, dK, dV


def rope_rotate(x, cos, sin) -> np.ndarray:
    """Rotary position embedding of x [B, L, H, d] with per-token angles given
    as cos, sin [L, d/2]: each adjacent pair (x_2i, x_2i+1) of token t turns by
    the angle phi_ti,
        x'_2i   = x_2i cos phi_ti - x_2i+1 sin phi_ti
        x'_2i+1 = x_2i sin phi_ti + x_2i+1 cos phi_ti.
    The pages name RoPE as the positional treatment of Q and K and as a neighbour
    of the attention inside the layer-level JVP (Causal-rCM summary page,
    section 3, "KV Cache": pre- and post-RoPE caching); they give no formula, so
    this is the standard rotary embedding on adjacent pairs, with the angles
    (1-D or 3-D positions, the packed clean|noisy order) left to the caller."""
    x = _as64(x)
    c = _as64(cos)[None, :, None, :]
    s = _as64(sin)[None, :, None, :]
    a, b = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def attn_jvp_rope_dense(q, k, v, tq, tk, tv, cos, sin, mode: int, c: int, n: int,
                        scale: Optional[float] = None, groups: Optional[Sequence[Group]] = None):
    """O, tO, LSE of the attention JVP with RoPE applied to the queries and keys
    first. The rotation does not depend on its input, so the tangents of the
    rotated queries and keys are the rotated tangents."""
    return attn_jvp_dense(rope_rotate(q, cos, sin), rope_rotate(k, cos, sin), v,
                          rope_rotate(tq, cos, sin), rope_rotate(tk, cos, sin), tv,
                          mode, c, n, scale, groups=groups)


def rope_angles_1d(L: int, d: int, base: float = 10000.0) -> Tuple[np.ndarray, np.ndarray]:
    """cos, sin [L, d/2] of 1-D positions 0..L-1 with frequencies base^(-2i/d)."""
    t = np.arange(L, dtype=np.float64)[:, None]
    theta = base ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)[None, :]
    return np.cos(t * theta), np.sin(t * theta)
