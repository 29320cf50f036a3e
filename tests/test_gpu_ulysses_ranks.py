"""Tangent-aware Ulysses context parallelism with the library's kernels as the
local attention and backward, on 2 and 3 ranks, checked against the oracle.

Causal-rCM summary page, section 3 "Parallelisms" and "KV Cache": the token
sequence is sharded across ranks; an all-to-all turns sequence shards of Q, K,
V (and, for the JVP, of tQ, tK, tV) into full-sequence shards of H/G heads,
each rank attends over its heads, and an all-to-all returns O, tO and LSE to
sequence shards. The backward is the transposed exchange around the backward
kernel.

Each rank is its own process. The exchange runs on a gloo process group over
host tensors; the `attn` and `bwd` callables move the rank's head shard to
cuda:0, run the library's forward+JVP or backward kernel there and move the
results back. The ranks' kernels never wait on one another (only the host
exchange synchronises them), so sharing one GPU between the rank processes is
safe. Every rank's O, tO, LSE, dQ, dK and dV are compared element by element
with the float64 oracle run on the whole, unsharded problem, at the parity
tolerances of the single-GPU tests: 2e-2 (1 + |ref|) for bf16 O, tO, dQ, dK,
dV and 1e-3 (1 + |ref|) for LSE.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _workload(case):
    from attention_jvp_attn_b200 import inputs as wl
    name, B, H, d, mask, seed = case
    if isinstance(mask, dict):
        # the group-table cases carry their length in the table; the workload
        # only draws the inputs (block-causal chunking of the same length)
        L = mask["groups"][-1][0]
        return wl.Workload(name, B=B, H=H, d=d, n_chunks=1, chunk_tokens=L, mode=wl.BLOCK_CAUSAL,
                           seed=seed)
    mode, c, n = mask
    return wl.Workload(name, B=B, H=H, d=d, n_chunks=n, chunk_tokens=c, mode=mode, seed=seed)


def _inputs(case):
    """Full-sequence bf16 inputs on the host and a seeded output cotangent dO."""
    from attention_jvp_attn_b200 import inputs as wl
    w = _workload(case)
    x = wl.make_inputs(w, device="cpu")
    g = torch.Generator().manual_seed(w.seed + 17)
    do = torch.randn(x["q"].shape, generator=g).to(torch.bfloat16)
    return w, [x[n] for n in wl.TENSOR_ORDER], do


def _gpu_attn(mask):
    import attention_jvp_attn_b200 as aj
    dev = torch.device("cuda", 0)

    def run(q, k, v, tq, tk, tv, scale):
        ins = [t.to(dev) for t in (q, k, v, tq, tk, tv)]
        if isinstance(mask, dict):
            o, to, lse = aj.attn_jvp_groups(*ins, mask["groups"], scale)
        else:
            o, to, lse = aj.attn_jvp(*ins, *mask, scale)
        if aj.sync_status(dev) != 0:
            raise RuntimeError("device status error")
        return o.cpu(), to.cpu(), lse.cpu()

    return run


def _gpu_bwd(mask):
    import attention_jvp_attn_b200 as aj
    dev = torch.device("cuda", 0)

    def run(q, k, v, o, do, lse, scale, dlse):
        ins = [t.to(dev) for t in (q, k, v, o, do)]
        lse_d = lse.to(dev)
        dlse_d = dlse.to(dev) if dlse is not None else None
        if isinstance(mask, dict):
            g = aj.attn_jvp_bwd_groups(*ins, lse_d, mask["groups"], scale, dlse=dlse_d)
        else:
            g = aj.attn_jvp_bwd(*ins, lse_d, *mask, scale, dlse=dlse_d)
        if aj.sync_status(dev) != 0:
            raise RuntimeError("device status error")
        return tuple(t.cpu() for t in g)

    return run


def _worker(rank, world, port, case, out_q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp, ulysses_attn_jvp_bwd
    torch.cuda.set_device(0)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        _, B, H, d, mask, seed = case
        w, full, do = _inputs(case)
        Ls = w.L // world
        sl = slice(rank * Ls, (rank + 1) * Ls)
        local = [t[:, sl].contiguous() for t in full]
        o, to, lse = ulysses_attn_jvp(*local, mask, None, attn=_gpu_attn(mask))
        # the backward starts from this rank's forward outputs, as in training
        dq, dk, dv = ulysses_attn_jvp_bwd(local[0], local[1], local[2], o, do[:, sl].contiguous(),
                                          lse, mask, None, bwd=_gpu_bwd(mask))
        out_q.put((rank,) + tuple(t.double().numpy() for t in (o, to, lse, dq, dk, dv)))
    finally:
        dist.destroy_process_group()


CASES = {
    # name, B, H, d, mask (mode, c, n) or {"groups": table}, seed
    # teacher forcing, L = 900: ragged last 256-row pair block and chunk edges inside tiles
    "tf_d128_2ranks": ("uly_tf", 1, 4, 128, (0, 150, 3), 611),
    # block causal, L = 384 split in three, B = 2, single-CTA d = 64 kernel
    "bc_d64_3ranks": ("uly_bc", 2, 6, 64, (1, 96, 4), 612),
    # sliding window of 200 keys as a group table over L = 512
    "window_d128_2ranks": ("uly_win", 1, 2, 128,
                           {"groups": [(r + 64, max(0, r + 64 - 200), r + 64, r + 64, r + 64)
                                       for r in range(0, 512, 64)]}, 613),
}
WORLD = {"tf_d128_2ranks": 2, "bc_d64_3ranks": 3, "window_d128_2ranks": 2}


def _close(got, ref, tol, what):
    err = np.abs(got - ref) / (1.0 + np.abs(ref))
    assert np.isfinite(got).all(), what
    assert err.max() <= tol, f"{what}: max scaled error {err.max():.3e} > {tol}"


@pytest.mark.parametrize("name", list(CASES))
def test_ulysses_ranks_with_kernels_match_oracle(cuda_device, name):
    from oracle import attn_jvp_oracle as orc
    world = WORLD[name]
    case = CASES[name]
    ctx = mp.get_context("spawn")
    out_q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, out_q))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    try:
        for _ in range(world):
            r, *outs = out_q.get(timeout=300)
            res[r] = outs
    finally:
        for p in procs:
            p.join(120)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)

    w, full, do = _inputs(case)
    mask = case[4]
    groups = mask["groups"] if isinstance(mask, dict) else None
    m = (0, 1, 1) if groups else mask
    O, tO, LSE = orc.attn_jvp_dense(*full, *m, None, groups=groups)
    dQ, dK, dV = orc.attn_vjp_dense(full[0], full[1], full[2], do, *m, None, groups=groups)
    Ls = w.L // world
    for r in range(world):
        sl = slice(r * Ls, (r + 1) * Ls)
        o, to, lse, dq, dk, dv = res[r]
        _close(o, O[:, sl], 2e-2, f"rank {r} O")
        _close(to, tO[:, sl], 2e-2, f"rank {r} tO")
        _close(lse, LSE[:, :, sl], 1e-3, f"rank {r} LSE")
        _close(dq, dQ[:, sl], 2e-2, f"rank {r} dQ")
        _close(dk, dK[:, sl], 2e-2, f"rank {r} dK")
        _close(dv, dV[:, sl], 2e-2, f"rank {r} dV")
