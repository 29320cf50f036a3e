"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The path shards into independent (batch, head, query-tile) units, so the only
cross-rank steps are the barrier and the MAX reduction of timings; every rank
draws its own replica of the inputs. These tests run those steps on two CPU
processes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    from attention_jvp_attn_b200 import inputs as wl
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        t = bench.max_over_ranks(10.0 + 5.0 * rank)          # per-rank "ms"
        seed = bench.rank_seed(wl.FRAMEWISE_TF, rank)
        x = wl.make_inputs(wl.TINY_F32, seed=seed)["q"]
        dist.barrier()
        q.put((rank, t, seed, float(x.flatten()[0])))
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_max_and_distinct_replicas():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    # every rank sees the slowest rank's time
    assert res[0][1] == 15.0 and res[1][1] == 15.0
    # the ranks draw different inputs
    assert res[0][2] != res[1][2] and res[0][3] != res[1][3]


def test_job_throughput_is_whole_job_over_slowest_rank():
    sys.path.insert(0, ROOT)
    import bench
    # 2 ranks x 3 steps x 1e12 FLOP in 1.5 s (slowest rank) = 4 TFLOP/s
    assert bench.job_throughput(2, 10**12, 3, 1500.0) == pytest.approx(4.0)
    assert bench.max_over_ranks(7.5) == 7.5  # no process group: identity


def test_reference_arm_other_ranks_exit_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "0"],
                       capture_output=True, text=True, env=env, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_prints_one_contract_line():
    # rank 0 of the reference arm: the oracle on a bounded sample, one JSON line
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0", "--ref-budget", "0.5"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "framewise_tf_bf16"
    # ms_per_step is the measured time of one bounded sample (about --ref-budget
    # seconds of oracle work), not an extrapolation to a full call
    assert 400.0 <= d["ms_per_step"] < 60000.0
    assert d["extrapolated_full_call_ms"] > d["ms_per_step"]


def test_bench_parity_leg_passes_on_oracle_outputs_and_catches_a_wrong_row():
    # the CPU-baseline leg compares the oracle on sampled rows with the timed
    # call's outputs; here the "GPU outputs" are the oracle's own, rounded to bf16
    sys.path.insert(0, ROOT)
    import torch
    import bench
    from attention_jvp_attn_b200 import inputs as wl
    from oracle import attn_jvp_oracle as orc
    w = wl.Workload("bench_parity", B=2, H=3, d=64, n_chunks=3, chunk_tokens=100, seed=3)
    x = wl.make_inputs(w)
    O, tO, L = orc.attn_jvp_dense(*(x[n] for n in wl.TENSOR_ORDER), w.mode, w.chunk_tokens,
                                  w.n_chunks)
    outs = (torch.from_numpy(O).bfloat16(), torch.from_numpy(tO).bfloat16(),
            torch.from_numpy(L).float())
    cpu, par = bench.oracle_check_and_time(w, x, outs, budget_s=0.3)
    assert par["pass"] and par["rows"] > 0 and cpu["kind"] == "oracle" and cpu["value"] > 0
    outs[1][1, 0, 2, 3] += 1.0  # row 0 of the last (batch, head) slice is always sampled
    _, par = bench.oracle_check_and_time(w, x, outs, budget_s=0.1)
    assert not par["pass"] and par["max_err_over_bound_tO"] > 1.0
