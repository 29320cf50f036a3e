"""Benchmark: custom-mask attention forward + JVP on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step is one call of the fused attention+JVP kernel over one batch of the
workload (default: frame-wise teacher forcing, B=1, H=12, d=128, 21 chunks x
1560 tokens packed clean|noisy, L=65520, bf16), inputs resident in HBM. The
metric is effective TFLOP/s over admissible (unmasked) query-key pairs,
12 d FLOPs per pair. Each rank runs its own replica of the workload (weak
scaling, no collective on the data path); rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle on the host cores instead (a
bounded sample of the same workload per step) and prints the same line.
Other modes, one JSON line each: --sweep (every sweep point), --backward (the
backward of the primal attention), --rope (the rotary embedding pass),
--ulysses (one problem sharded by heads over the ranks, strong scaling).
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}
METRIC = "attention+JVP effective TFLOP/s (unmasked pairs) and % of B200 bf16 peak"
RANK_SEED_STRIDE = 7919


def rank_seed(w, rank: int) -> int:
    """Seed of a rank's replica of the workload (replicas draw different inputs)."""
    return w.seed + RANK_SEED_STRIDE * rank


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a per-rank timing over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job TFLOP/s: every rank ran `steps` steps; time is the slowest rank's."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


def _env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    """Hash of the sources the forward kernels are built from (the backward's
    and the rotary embedding's own source files do not change them)."""
    h = hashlib.sha256()
    for p in sorted(glob.glob(os.path.join(ROOT, "attention_jvp_attn_b200", "csrc", "*"))):
        if os.path.basename(p).startswith(("attn_jvp_bwd", "attn_jvp_rope")):
            continue
        with open(p, "rb") as f:
            h.update(os.path.basename(p).encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("kernel_hash") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            self.proc.wait()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        power = [num(r[3]) for r in rows if num(r[3]) is not None]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(power) if power else None}


def workload_by_name(name, heads=None):
    from attention_jvp_attn_b200 import inputs as wl
    if name not in wl.WORKLOADS:
        raise SystemExit(f"unknown workload {name}; choose from {sorted(wl.WORKLOADS)}")
    w = wl.WORKLOADS[name]
    if heads is not None:
        w = w.with_(H=heads, name=f"{w.name}_h{heads}")
    return w


def flops_per_step(w) -> int:
    from attention_jvp_attn_b200 import inputs as wl
    c, n = w.chunk_tokens, w.n_chunks
    pairs = c * c * n * (n + 1) // (1 if w.mode == wl.TEACHER_FORCING else 2)
    return 12 * w.d * pairs * w.B * w.H


def workload_config(w, n_gpus):
    from attention_jvp_attn_b200 import inputs as wl
    return {"workload": w.name, "mask": wl.MODE_NAMES[w.mode], "B": w.B, "H": w.H, "d": w.d,
            "n_chunks": w.n_chunks, "chunk_tokens": w.chunk_tokens, "seq_len": w.L,
            "global_batch": w.B * n_gpus, "parallelism": f"{n_gpus} independent replicas",
            "l2": f"no flush: inputs {w.input_bytes() / 1e9:.2f} GB > 126 MB L2"}


# --------------------------------------------------------------------------- oracle timing

def _oracle_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=1)
    except Exception:
        return 1


def _timed_oracle_rows(w, x64, rows):
    """The float64 oracle on query rows `rows` of one (batch, head) whose [L, d]
    inputs are x64: (O, tO, LSE of the rows, seconds, admissible pairs)."""
    import numpy as np
    from oracle import attn_jvp_oracle as orc
    rows = np.asarray(rows, dtype=np.int64)
    t0 = time.perf_counter()
    O, tO, lse = orc.attn_jvp_rows(*x64, w.mode, w.chunk_tokens, w.n_chunks, w.scale, rows)
    secs = time.perf_counter() - t0
    M = orc.allowed(w.mode, w.chunk_tokens, w.n_chunks, rows[:, None], np.arange(w.L)[None, :])
    return O, tO, lse, secs, int(M.sum())


def oracle_sample(w, budget_s: float, seed: int = 0):
    """Time the float64 oracle on seeded random query rows of head 0 of the
    workload (CPU inputs drawn from the same generator recipe), growing the
    sample until about `budget_s` seconds of work. Returns (effective FLOP/s,
    rows, seconds, threads)."""
    import numpy as np
    import torch
    from oracle import attn_jvp_oracle as orc
    g = torch.Generator().manual_seed(w.seed)
    one = (w.L, w.d)
    x = [(torch.randn(one, generator=g) * s).to(torch.bfloat16 if w.dtype == "bf16" else torch.float32)
         for s in w.stds]
    x64 = [orc._as64(t) for t in x]
    rng = np.random.default_rng(seed)
    total_pairs, total_t, rows_done = 0, 0.0, 0
    batch = 16
    while total_t < budget_s:
        rows = rng.integers(0, w.L, size=batch)
        _, _, _, t, pairs = _timed_oracle_rows(w, x64, rows)
        total_t += t
        total_pairs += pairs
        rows_done += batch
        if total_t < budget_s / 4:
            batch = min(2 * batch, 4096)
    return 12 * w.d * total_pairs / total_t, rows_done, total_t, _oracle_threads()


def oracle_check_and_time(w, x, outs, budget_s: float, seed: int = 0):
    """The CPU-baseline leg on the timed call's own data: the float64 oracle
    on sampled query rows of two (batch, head) slices of the GPU inputs `x`,
    timed, and its O, tO, LSE compared with the GPU outputs `outs` of the
    timed call on the same rows. Rows: every chunk's first and last row, the
    rows on both sides of the 128- and 256-row tile edges around chunk
    boundaries, the ragged tail and 64 seeded random rows per slice; then
    seeded random rows of the first slice until about `budget_s` seconds of
    oracle work. Returns (cpu_baseline dict, parity dict)."""
    import numpy as np
    from attention_jvp_attn_b200 import inputs as wl
    from oracle import attn_jvp_oracle as orc
    o, to, lse = outs
    tol = 2e-2 if w.dtype == "bf16" else 1e-4
    tol_lse = 1e-3 if w.dtype == "bf16" else 1e-4
    struct = sorted(set(wl.sample_rows(w, n_random=64, seed=seed + 11, tile=128)) |
                    set(wl.sample_rows(w, n_random=0, tile=256)))
    slices = [(0, 0), (w.B - 1, w.H - 1)]
    worst = {"O": 0.0, "tO": 0.0, "LSE": 0.0}
    total_t, total_pairs, n_rows = 0.0, 0, 0
    rng = np.random.default_rng(seed)

    def check(b, h, x64, rows):
        nonlocal total_t, total_pairs, n_rows
        O, tO, L_, t, pairs = _timed_oracle_rows(w, x64, rows)
        total_t += t
        total_pairs += pairs
        n_rows += len(rows)
        idx = np.asarray(rows)
        got = (o[b, idx, h].double().cpu().numpy(), to[b, idx, h].double().cpu().numpy(),
               lse[b, h, idx].double().cpu().numpy())
        for name, g, r, tl in (("O", got[0], O, tol), ("tO", got[1], tO, tol),
                               ("LSE", got[2], L_, tol_lse)):
            ratio = np.abs(g - r) / (tl * (1.0 + np.abs(r)))
            worst[name] = max(worst[name], float(np.nanmax(ratio)) if np.isfinite(g).all()
                              else float("inf"))

    first = None
    for b, h in slices:
        x64 = [orc._as64(x[n][b, :, h]) for n in wl.TENSOR_ORDER]
        first = first or (b, h, x64)
        check(b, h, x64, struct)
    b, h, x64 = first
    batch = 16
    while total_t < budget_s:
        check(b, h, x64, sorted(set(rng.integers(0, w.L, size=batch).tolist())))
        if total_t < budget_s / 4:
            batch = min(2 * batch, 4096)
    cpu = {"value": 12 * w.d * total_pairs / total_t / 1e12, "unit": "TFLOP/s",
           "cores": _oracle_threads(), "kind": "oracle",
           "sample": (f"{n_rows} query rows of (batch, head) slices {slices} of the timed "
                      f"call's inputs (chunk and tile edges, ragged tail, seeded random rows), "
                      f"{total_t:.1f} s of float64 oracle work; effective FLOPs = 12 d x "
                      f"admissible pairs of those rows")}
    parity = {"rows": n_rows, "slices": [list(s) for s in slices],
              "bound": f"|err| <= {tol} (1 + |ref|) for O and tO, {tol_lse} (1 + |ref|) for LSE",
              "max_err_over_bound_O": worst["O"], "max_err_over_bound_tO": worst["tO"],
              "max_err_over_bound_LSE": worst["LSE"],
              "pass": all(v <= 1.0 for v in worst.values())}
    return cpu, parity


def run_reference(args):
    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    if rank != 0:
        return 0
    w = workload_by_name(args.workload, args.heads)
    for _ in range(args.warmup):
        oracle_sample(w, budget_s=0.5)
    vals, secs, rows_all = [], 0.0, 0
    threads = 1
    t_steps = time.perf_counter()
    for _ in range(args.steps):
        v, rows, t, threads = oracle_sample(w, budget_s=args.ref_budget)
        vals.append(v)
        secs += t
        rows_all += rows
    wall_s = time.perf_counter() - t_steps
    value = statistics.mean(vals) / 1e12
    sample = (f"{rows_all} seeded random query rows of head 0 over {args.steps} steps "
              f"(about {args.ref_budget:.0f} s each), float64 dense rows masked by the explicit "
              f"predicate; effective FLOPs = 12 d x admissible pairs of the sampled rows")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * wall_s / args.steps,
            "step": "one bounded sample of query rows of the workload (not a full call)",
            "extrapolated_full_call_ms": 1e3 * flops_per_step(w) / (value * 1e12),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, 1),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0




# --------------------------------------------------------------------------- GPU arm

def run_gpu(args):
    import torch
    import torch.distributed as dist
    import attention_jvp_attn_b200 as aj
    from attention_jvp_attn_b200 import inputs as wl

    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    local = _env_int("LOCAL_RANK", 0)
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    w = workload_by_name(args.workload, args.heads)
    x = wl.make_inputs(w, device=dev, seed=rank_seed(w, rank))
    B, L, H, d = w.B, w.L, w.H, w.d
    dt = x["q"].dtype
    o = torch.empty_like(x["q"])
    to = torch.empty_like(x["q"])
    lse = torch.empty((B, H, L), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode, w.chunk_tokens,
                    w.n_chunks, w.scale, out=(o, to, lse))

    for _ in range(max(args.warmup, 0)):
        step()
    st = aj.sync_status(dev)
    if st != 0:
        raise SystemExit(f"device status {st} after warm-up")

    clocks = ClockSampler(local)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.25)  # let the sampler start before the timed region
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(args.steps):
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    st = aj.sync_status(dev)
    if st != 0:
        raise SystemExit(f"device status {st} after timed steps")
    total_ms = t_begin.elapsed_time(t_end)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(total_ms, dev)
    ms_per_step = total_ms / args.steps
    flops = flops_per_step(w)
    value = job_throughput(world, flops, args.steps, total_ms)

    # end to end through the host-buffer C-ABI entry point (pinned host memory)
    e2e = None
    e2e_steps = args.e2e_steps if args.e2e_steps is not None else args.steps
    if not args.no_e2e:
        xh = {k: v.cpu().pin_memory() for k, v in x.items()}
        oh = torch.empty((B, L, H, d), dtype=dt).pin_memory()
        toh = torch.empty((B, L, H, d), dtype=dt).pin_memory()
        lseh = torch.empty((B, H, L), dtype=torch.float32).pin_memory()
        staging = torch.empty(aj.host_staging_bytes(B, L, H, d, dt), dtype=torch.uint8, device=dev)

        def e2e_step():
            aj.attn_jvp_host(xh["q"], xh["k"], xh["v"], xh["tq"], xh["tk"], xh["tv"], w.mode,
                             w.chunk_tokens, w.n_chunks, staging, (oh, toh, lseh), w.scale, dev)
        e2e_step()
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        tensor_bytes = B * L * H * d * x["q"].element_size()
        e2e = {"value": job_throughput(world, flops, e2e_steps, e2e_ms), "unit": "TFLOP/s",
               "ms_per_step": e2e_ms / e2e_steps, "steps": e2e_steps,
               "h2d_bytes_per_step": 6 * tensor_bytes,
               "d2h_bytes_per_step": 2 * tensor_bytes + B * H * L * 4}
        del xh, oh, toh, lseh, staging

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    avg_launch_ms = sum(launch_ms) / len(launch_ms)
    achieved = flops / (avg_launch_ms * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": load_traffic(w.name),
                "peak_source": f"{peak_src} bf16 dense burst",
                "sustained_peak": float(peaks.get("bf16_tflops_sustained",
                                                  FALLBACK_PEAKS["bf16_tflops_sustained"])),
                "kernel": "attn_jvp_tc_kernel<128, true> (CTA pairs)" if d == 128 else "attn_jvp_tc_kernel<64, false>",
                "flops_per_launch": flops, "avg_launch_ms": avg_launch_ms}
    cpu, parity = None, None
    if world == 1 and not args.no_cpu_baseline:
        cpu, parity = oracle_check_and_time(w, x, (o, to, lse), budget_s=args.cpu_budget)
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "pct_of_peak": 100.0 * value / world / peak,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": workload_config(w, world), "roofline": roofline, "cpu_baseline": cpu,
            "e2e": e2e, "parity": parity, "gpu_launches": args.steps, "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def run_ulysses(args) -> int:
    """Head-sharded (Ulysses) attention JVP over the process group: each rank
    holds one sequence block [B, L/N, H, d] of the six inputs of the same
    problem; an NCCL all-to-all turns them into full-sequence shards of H/N
    heads, the kernel runs on them, and all-to-alls return O, tO and LSE to
    sequence blocks. The whole problem is fixed as N grows ("strong"
    scaling); value = the problem's effective FLOPs per step x steps / the
    slowest rank's time. With one rank the exchange is the identity."""
    import socket
    import torch
    import torch.distributed as dist
    import attention_jvp_attn_b200 as aj
    from attention_jvp_attn_b200 import inputs as wl
    from attention_jvp_attn_b200.ulysses import ulysses_attn_jvp

    rank = _env_int("RANK", 0)
    world = _env_int("WORLD_SIZE", 1)
    local = _env_int("LOCAL_RANK", 0)
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = workload_by_name(args.workload, args.heads)
    if w.H % world or w.L % world:
        raise SystemExit(f"--ulysses needs H ({w.H}) and L ({w.L}) divisible by {world} ranks")
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    else:
        with socket.socket() as sk:
            sk.bind(("127.0.0.1", 0))
            port = sk.getsockname()[1]
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                                world_size=1, timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    full = wl.make_inputs(w, device=dev)
    Ls = w.L // world
    x = [full[n][:, rank * Ls:(rank + 1) * Ls].contiguous() for n in wl.TENSOR_ORDER]
    del full
    torch.cuda.empty_cache()
    mask = (w.mode, w.chunk_tokens, w.n_chunks)
    stream = torch.cuda.current_stream(dev)

    def step():
        return ulysses_attn_jvp(*x, mask, w.scale)

    for _ in range(max(args.warmup, 1)):
        step()
    st = aj.sync_status(dev)
    if st != 0:
        raise SystemExit(f"device status {st} after warm-up")
    clocks = ClockSampler(local)
    dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    time.sleep(0.25)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    st = aj.sync_status(dev)
    if st != 0:
        raise SystemExit(f"device status {st} after timed steps")
    total_ms = max_over_ranks(t0.elapsed_time(t1), dev)
    dist.barrier()
    dist.destroy_process_group()
    if rank != 0:
        return 0
    flops = flops_per_step(w)
    value = flops * args.steps / (total_ms * 1e-3) / 1e12
    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    cfg = workload_config(w, world)
    cfg["parallelism"] = f"Ulysses head sharding over {world} ranks (NCCL all-to-all)"
    cfg["global_batch"] = w.B
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "pct_of_peak": 100.0 * value / world / peak,
            "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic",
            "config": cfg, "mode": "ulysses", "gpu_launches": args.steps, "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def run_sweep(args) -> int:
    """Sweep (config 5): every point of inputs.sweep_points() on one GPU, one
    JSON line each (CUDA-event median of `--steps` launches after `--warmup`),
    then a summary line. Device timing only; inputs resident."""
    import torch
    import attention_jvp_attn_b200 as aj
    from attention_jvp_attn_b200 import inputs as wl
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--sweep runs on one GPU")
    dev = torch.device("cuda", 0)
    peaks, _ = load_peaks()
    peak = peaks["bf16_tflops"]
    rows = []
    for w in wl.sweep_points():
        x = wl.make_inputs(w, device=dev)
        o = torch.empty_like(x["q"])
        to = torch.empty_like(x["q"])
        lse = torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev)

        def step():
            aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode,
                        w.chunk_tokens, w.n_chunks, w.scale, out=(o, to, lse))

        for _ in range(max(args.warmup, 1)):
            step()
        if aj.sync_status(dev) != 0:
            raise SystemExit(f"device status error on {w.name}")
        ms = []
        for _ in range(args.steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize(dev)
            ms.append(e0.elapsed_time(e1))
        ms.sort()
        med = ms[len(ms) // 2]
        tf = flops_per_step(w) / (med * 1e-3) / 1e12
        row = {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d,
               "chunk_tokens": w.chunk_tokens, "n_chunks": w.n_chunks, "ms": med,
               "tflops": tf, "pct_of_peak": 100.0 * tf / peak}
        rows.append(row)
        print(json.dumps(row), flush=True)
        del x, o, to, lse
        torch.cuda.empty_cache()
    tfs = sorted(r["tflops"] for r in rows)
    print(json.dumps({"sweep_points": len(rows), "tflops_min": tfs[0], "tflops_median": tfs[len(tfs) // 2],
                      "tflops_max": tfs[-1], "unit": "TFLOP/s", "peak": peak}), flush=True)
    return 0


def run_backward(args) -> int:
    """Backward of the primal attention (attn_jvp_bwd) on one GPU: dQ, dK, dV
    from the workload's Q, K, V, the forward's O and LSE and a seeded random
    cotangent dO. One JSON line: CUDA-event median over `--steps` calls after
    `--warmup`, inputs resident. Effective FLOPs count 10 d per admissible
    pair (the products S, dP, dV, dK, dQ at 2 d each). For bf16 the call runs
    on the tensor cores in three launches (row statistics, then dK/dV per key
    block, then dQ per query block); S and dP are formed in both the dK/dV
    and the dQ kernel, so 14 d FLOPs per pair execute. The roofline peak is
    the measured bf16 dense burst. fp32 runs on CUDA cores against a peak of
    148 SMs x 128 fp32 lanes x 2 FLOPs x the sampled SM clock."""
    import torch
    import attention_jvp_attn_b200 as aj
    from attention_jvp_attn_b200 import inputs as wl
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--backward runs on one GPU")
    dev = torch.device("cuda", 0)
    w = workload_by_name(args.workload, args.heads)
    x = wl.make_inputs(w, device=dev)
    o, _, lse = aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode,
                            w.chunk_tokens, w.n_chunks, w.scale)
    del x["tq"], x["tk"], x["tv"]
    g = torch.Generator(device=dev).manual_seed(1234)
    do = torch.randn(x["q"].shape, generator=g, device=dev).to(x["q"].dtype)
    out = tuple(torch.empty_like(x["q"]) for _ in range(3))

    def step():
        aj.attn_jvp_bwd(x["q"], x["k"], x["v"], o, do, lse, w.mode, w.chunk_tokens, w.n_chunks,
                        w.scale, out=out)

    for _ in range(max(args.warmup, 1)):
        step()
    if aj.sync_status(dev) != 0:
        raise SystemExit("device status error")
    clocks = ClockSampler(0)
    clocks.start()
    ms = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        step()
        e1.record()
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1))
    ck = clocks.stop()
    if aj.sync_status(dev) != 0:
        raise SystemExit("device status error")
    ms.sort()
    med = ms[len(ms) // 2]
    pairs_total = flops_per_step(w) // (12 * w.d)
    eff = 10 * w.d * pairs_total / (med * 1e-3) / 1e12
    if w.dtype == "bf16":
        peaks, kind = load_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        executed = 14 * w.d * pairs_total / (med * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": eff, "peak": peak, "unit": "TFLOP/s",
                "frac": eff / peak, "peak_source": f"{kind} bf16 dense burst",
                "executed_tflops": executed, "executed_frac": executed / peak,
                "note": "achieved counts 10 d per pair; 14 d execute (S, dP in both kernels)",
                "kernels": ["bwd_prep_kernel", "bwd_dkdv_tc_kernel", "bwd_dq_tc_kernel"]}
    else:
        executed = 14 * w.d * pairs_total / (med * 1e-3) / 1e12
        mhz = (ck or {}).get("sm_mhz") or 1965.0
        alu_peak = 148 * 128 * 2 * mhz * 1e6 / 1e12
        roof = {"bound": "alu", "achieved": executed, "peak": alu_peak, "unit": "TFLOP/s",
                "frac": executed / alu_peak,
                "note": "fp32 FMA pipe; 14 d FLOPs executed per pair"}
    print(json.dumps({"mode": "backward", "workload": w.name, "dtype": w.dtype,
                      "B": w.B, "H": w.H, "L": w.L, "d": w.d, "steps": args.steps,
                      "warmup": args.warmup, "ms": med, "ms_min": ms[0], "ms_max": ms[-1],
                      "metric": "backward effective TFLOP/s (10 d per admissible pair)",
                      "value": eff, "unit": "TFLOP/s", "roofline": roof,
                      "clocks": ck}), flush=True)
    return 0


def run_rope(args) -> int:
    """Rotary embedding of Q, K, tQ, tK on one GPU, one JSON line.

    - The stand-alone pass (attn_jvp_rope in C, `rope` in Python): HBM-bound;
      algorithmic bytes are the four tensors read and written plus the cos/sin
      tables read once. Timed over `--rope-calls` back-to-back calls, so that the
      timed region spans several clock samples.
    - The fused call (attn_jvp_fwd_rope: rotation and attention in one launch
      for bf16) against attn_jvp alone on the same inputs: the CUDA-event
      median of `--steps` calls each, after `--warmup`.
    Inputs are resident (each tensor larger than L2)."""
    import numpy as np
    import torch
    import attention_jvp_attn_b200 as aj
    from attention_jvp_attn_b200 import inputs as wl
    if int(os.environ.get("WORLD_SIZE", "1")) > 1:
        raise SystemExit("--rope runs on one GPU")
    dev = torch.device("cuda", 0)
    w = workload_by_name(args.workload, args.heads)
    x = wl.make_inputs(w, device=dev)
    phi = np.random.default_rng(0).uniform(-np.pi, np.pi, (w.L, w.d // 2))
    cos = torch.from_numpy(np.cos(phi).astype(np.float32)).to(dev)
    sin = torch.from_numpy(np.sin(phi).astype(np.float32)).to(dev)
    ins = (x["q"], x["k"], x["tq"], x["tk"])
    rot = tuple(torch.empty_like(t) for t in ins)

    def rope_step():
        aj.rope(*ins, cos, sin, out=rot)

    for _ in range(max(args.warmup, 1)):
        rope_step()
    if aj.sync_status(dev) != 0:
        raise SystemExit("device status error")
    clocks = ClockSampler(0)
    clocks.start()
    time.sleep(0.25)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.rope_calls):
        rope_step()
    e1.record()
    torch.cuda.synchronize(dev)
    ck = clocks.stop()
    if aj.sync_status(dev) != 0:
        raise SystemExit("device status error")
    ms = e0.elapsed_time(e1) / args.rope_calls
    tensor_bytes = ins[0].numel() * ins[0].element_size()
    alg = 8 * tensor_bytes + 2 * cos.numel() * 4
    peaks, kind = load_peaks()
    gbs = alg / (ms * 1e-3) / 1e9

    outs = (torch.empty_like(x["q"]), torch.empty_like(x["q"]),
            torch.empty((w.B, w.H, w.L), dtype=torch.float32, device=dev))

    def fused_step():
        aj.attn_jvp_rope(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], cos, sin, w.mode,
                         w.chunk_tokens, w.n_chunks, w.scale, out=outs, rotated=rot)

    def plain_step():
        aj.attn_jvp(x["q"], x["k"], x["v"], x["tq"], x["tk"], x["tv"], w.mode, w.chunk_tokens,
                    w.n_chunks, w.scale, out=outs)

    def median_ms(fn):
        for _ in range(max(args.warmup, 1)):
            fn()
        t = []
        for _ in range(args.steps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize(dev)
            t.append(a.elapsed_time(b))
        t.sort()
        return t[len(t) // 2]

    clocks2 = ClockSampler(0)
    clocks2.start()
    fused_ms = median_ms(fused_step)
    plain_ms = median_ms(plain_step)
    ck2 = clocks2.stop()
    if aj.sync_status(dev) != 0:
        raise SystemExit("device status error")
    print(json.dumps({"mode": "rope", "workload": w.name, "dtype": w.dtype, "B": w.B, "H": w.H,
                      "L": w.L, "d": w.d, "calls": args.rope_calls, "ms": ms,
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                                   "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                                   "algorithmic_bytes": alg, "peak_kind": kind},
                      "clocks": ck,
                      "fused": {"ms": fused_ms, "forward_alone_ms": plain_ms,
                                "overhead_pct": 100.0 * (fused_ms - plain_ms) / plain_ms,
                                "steps": args.steps, "clocks": ck2}}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="framewise_tf_bf16")
    ap.add_argument("--heads", type=int, default=None, help="override H (profiling a smaller case)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="timed steps of the end-to-end leg (default: --steps)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-budget", type=float, default=6.0)
    ap.add_argument("--sweep", action="store_true",
                    help="time every sweep point (config 5) on one GPU, one JSON line each")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward of the primal attention on one GPU (one JSON line)")
    ap.add_argument("--rope", action="store_true",
                    help="time the rotary embedding of Q, K, tQ, tK on one GPU (one JSON line)")
    ap.add_argument("--rope-calls", type=int, default=400,
                    help="calls of the stand-alone rotation timed back to back (--rope)")
    ap.add_argument("--ulysses", action="store_true",
                    help="one problem sharded over the ranks by heads (NCCL all-to-all; strong scaling)")
    args = ap.parse_args()
    if args.warmup < 0 or args.steps < 1:
        raise SystemExit("need --steps >= 1 and --warmup >= 0")
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    if args.backward:
        return run_backward(args)
    if args.rope:
        return run_rope(args)
    if args.ulysses:
        return run_ulysses(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
