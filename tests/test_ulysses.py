"""Tangent-aware Ulysses exchange (seq -> heads -> seq) on CPU ranks (gloo).

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
