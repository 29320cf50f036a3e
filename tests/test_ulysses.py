"""Tangent-aware Ulysses exchange (seq -> heads -> seq) on CPU ranks (gloo),
for the attention JVP and for the backward of the primal attention.

Each rank holds one sequence block of Q, K, V, tQ, tK, tV; after the
exchange it runs the attention JVP for its heads over the full sequence and
the outputs go back to sequence blocks. With the float64 oracle as the local
attention, every rank's O, tO and LSE must equal the matching slice of the
oracle run on the whole, unsharded problem, bit for bit: only data movement
happens around it.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_attn(mask):
    from oracle import attn_jvp_oracle as orc

    def run(q, k, v, tq, tk, tv, scale):
        if isinstance(mask, dict):
            O, tO, lse = orc.attn_jvp_dense(q, k, v, tq, tk, tv, 0, 1, 1, scale,
                                            groups=mask["groups"])
        else:
            O, tO, lse = orc.attn_jvp_dense(q, k, v, tq, tk, tv, *mask, scale)
        return torch.from_numpy(O), torch.from_numpy(tO), torch.from_numpy(lse)

    return run


def _full_inputs(B, L, H, d, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn((B, L, H, d), generator=g, dtype=torch.float64) for _ in range(6)]


def _worker(rank, world, port, case, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, L, H, d, mask, scale, seed = case
        full = _full_inputs(B, L, H, d, seed)
        Ls = L // world
        local = [t[:, rank * Ls:(rank + 1) * Ls].contiguous() for t in full]
        o, to, lse = ulysses_attn_jvp(*local, mask, scale, attn=_oracle_attn(mask))
        q.put((rank, o.numpy(), to.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


def _run(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, o, to, lse = q.get(timeout=120)
        res[r] = (o, to, lse)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    return res


CASES = {
    # B, L, H, d, mask, scale, seed
    "tf_2ranks": (2, 12, 6, 8, (0, 3, 2), None, 1),
    "bc_3ranks": (1, 12, 6, 4, (1, 4, 3), 0.3, 2),
    "groups_2ranks": (1, 16, 4, 8, {"groups": [(4, 0, 4, 4, 4), (10, 2, 6, 9, 12), (16, 0, 1, 8, 16)]},
                      None, 3),
}
WORLD = {"tf_2ranks": 2, "bc_3ranks": 3, "groups_2ranks": 2}


@pytest.mark.parametrize("name", list(CASES))
def test_ulysses_exchange_matches_unsharded_oracle(name):
    from oracle import attn_jvp_oracle as orc
    world = WORLD[name]
    case = CASES[name]
    B, L, H, d, mask, scale, seed = case
    res = _run(world, case)
    full = _full_inputs(B, L, H, d, seed)
    if isinstance(mask, dict):
        O, tO, LSE = orc.attn_jvp_dense(*full, 0, 1, 1, scale, groups=mask["groups"])
    else:
        O, tO, LSE = orc.attn_jvp_dense(*full, *mask, scale)
    Ls = L // world
    for r in range(world):
        o, to, lse = res[r]
        assert np.array_equal(o, O[:, r * Ls:(r + 1) * Ls])
        assert np.array_equal(to, tO[:, r * Ls:(r + 1) * Ls])
        assert np.array_equal(lse, LSE[:, :, r * Ls:(r + 1) * Ls])


def _mask_matrix(mask):
    from oracle import attn_jvp_oracle as orc
    if isinstance(mask, dict):
        return orc.mask_matrix_groups(mask["groups"])
    return orc.mask_matrix(*mask)


def _lse_based_bwd(mask):
    """Float64 backward that, like the kernel, rebuilds P from the LSE it is
    given and takes D_i from the O it is given, so a misplaced O or LSE row
    changes the result. Per (batch, head) 2-D products: the same bits whatever
    heads a rank holds."""
    M = _mask_matrix(mask)

    def run(q, k, v, o, do, lse, scale, dlse):
        B, L, H, d = q.shape
        s = 1.0 / np.sqrt(d) if scale is None else scale
        outs = [np.zeros((B, L, H, d)) for _ in range(3)]
        for b in range(B):
            for h in range(H):
                qq, kk, vv, oo, dd = (t[b, :, h].numpy() for t in (q, k, v, o, do))
                P = np.where(M, np.exp(s * (qq @ kk.T) - lse[b, h].numpy()[:, None]), 0.0)
                D = (dd * oo).sum(axis=1) - (dlse[b, h].numpy() if dlse is not None else 0.0)
                dS = P * (dd @ vv.T - D[:, None])
                outs[0][b, :, h] = s * (dS @ kk)
                outs[1][b, :, h] = s * (dS.T @ qq)
                outs[2][b, :, h] = P.T @ dd
        return tuple(torch.from_numpy(t) for t in outs)

    return run


def _bwd_full(case):
    from oracle import attn_jvp_oracle as orc
    B, L, H, d, mask, scale, seed = case
    q, k, v, do, _, _ = _full_inputs(B, L, H, d, seed)
    if isinstance(mask, dict):
        O, LSE = orc.attn_forward_dense(q, k, v, 0, 1, 1, scale, groups=mask["groups"])
    else:
        O, LSE = orc.attn_forward_dense(q, k, v, *mask, scale)
    dlse = torch.randn((B, H, L), generator=torch.Generator().manual_seed(seed + 1),
                       dtype=torch.float64)
    return q, k, v, torch.from_numpy(O), do, torch.from_numpy(LSE), dlse


def _bwd_worker(rank, world, port, case, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp_bwd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        B, L, H, d, mask, scale, seed = case
        qq, k, v, o, do, lse, dlse = _bwd_full(case)
        Ls = L // world
        sl = slice(rank * Ls, (rank + 1) * Ls)
        local = [t[:, sl].contiguous() for t in (qq, k, v, o, do)]
        out = ulysses_attn_jvp_bwd(*local, lse[:, :, sl].contiguous(), mask, scale,
                                   dlse=dlse[:, :, sl].contiguous(), bwd=_lse_based_bwd(mask))
        q.put((rank,) + tuple(t.numpy() for t in out))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", list(CASES))
def test_ulysses_backward_matches_unsharded(name):
    from oracle import attn_jvp_oracle as orc
    world = WORLD[name]
    case = CASES[name]
    B, L, H, d, mask, scale, seed = case
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, case, q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, *g = q.get(timeout=120)
        res[r] = g
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    qq, k, v, o, do, lse, dlse = _bwd_full(case)
    whole = [t.numpy() for t in _lse_based_bwd(mask)(qq, k, v, o, do, lse, scale, dlse)]
    groups = mask["groups"] if isinstance(mask, dict) else None
    m = (0, 1, 1) if groups else mask
    ref = orc.attn_vjp_dense(qq, k, v, do, *m, scale, dlse=dlse.numpy(), groups=groups)
    Ls = L // world
    for r in range(world):
        for got, full, exact in zip(res[r], whole, ref):
            # bit-equal to the same backward on the unsharded problem
            assert np.array_equal(got, full[:, r * Ls:(r + 1) * Ls])
            # and equal to the oracle's VJP up to float64 rounding
            np.testing.assert_allclose(got, exact[:, r * Ls:(r + 1) * Ls], rtol=1e-9, atol=1e-11)


def test_ulysses_rejects_a_mask_of_another_length():
    import torch.distributed as dist
    from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp
    port = _free_port()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        x = [torch.zeros(1, 8, 3, 4, dtype=torch.float64) for _ in range(6)]
        with pytest.raises(ValueError):
            ulysses_attn_jvp(*x, (1, 2, 3), None, attn=_oracle_attn((1, 2, 3)))  # L=8 vs 6
    finally:
        dist.destroy_process_group()


def test_ulysses_backward_rejects_bad_arguments():
    import torch.distributed as dist
    from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp_bwd
    port = _free_port()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=0, world_size=1)
    try:
        mask = (1, 2, 3)  # block causal, L = 6
        x = [torch.zeros(1, 6, 3, 4, dtype=torch.float64) for _ in range(5)]
        lse = torch.zeros(1, 3, 6, dtype=torch.float64)
        bwd = _lse_based_bwd(mask)
        with pytest.raises(ValueError):  # LSE of another length
            ulysses_attn_jvp_bwd(*x, torch.zeros(1, 3, 5, dtype=torch.float64), mask, bwd=bwd)
        with pytest.raises(ValueError):  # dLSE of another shape
            ulysses_attn_jvp_bwd(*x, lse, mask, dlse=torch.zeros(1, 2, 6, dtype=torch.float64),
                                 bwd=bwd)
        with pytest.raises(ValueError):  # mask of another length
            ulysses_attn_jvp_bwd(*x, lse, (1, 2, 2), bwd=bwd)
        with pytest.raises(ValueError):  # inputs of different shapes
            ulysses_attn_jvp_bwd(*x[:4], torch.zeros(1, 6, 3, 5, dtype=torch.float64), lse, mask,
                                 bwd=bwd)
        out = ulysses_attn_jvp_bwd(*x, lse, mask, bwd=bwd)  # and the valid call runs
        assert all(t.shape == (1, 6, 3, 4) for t in out)
    finally:
        dist.destroy_process_group()
