"""The benchmark's multi-rank host logic on CPU: world size 2 over gloo.

Each rank quantizes its own independent layer (weak scaling, no data-path
collective); the job's time is the slowest rank's, found by one MAX
all-reduce; rank 0 alone reports.  The GPU runs use NCCL for the same
calls; here the ranks are CPU processes with the gloo backend.
"""
import json
import multiprocessing as mp
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=timedelta(seconds=60))
    try:
        ms = 10.0 + 5.0 * rank           # rank 1 is the slow one
        ms_max = bench.max_over_ranks(ms, world, torch.device("cpu"))
        spec = bench.workload_spec("q_proj", rank)
        value = bench.weak_value(world, spec.d_row * spec.d_col, ms_max)
        q.put((rank, ms_max, spec.w_seed, spec.x_seed, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_distinct_layers():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, m0, w0, x0, v0), (r1, m1, w1, x1, v1) = res
    assert m0 == m1 == 15.0                      # every rank sees the max
    assert v0 == v1 == pytest.approx(2 * 4096 * 4096 / 15e-3)
    assert (w0, x0) != (w1, x1)                  # independent layers per rank


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, None) == 3.5
    assert bench.weak_value(1, 200, 2.0) == pytest.approx(100000.0)


def _reference_arm(rank, world):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--workload", "small", "--steps", "1", "--warmup", "0",
                           "--gpus", str(world)],
                          capture_output=True, text=True, env=env, timeout=300, cwd=ROOT)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _reference_arm(1, 2)
    assert r1.returncode == 0 and r1.stdout.strip() == ""
    r0 = _reference_arm(0, 2)
    assert r0.returncode == 0
    lines = [ln for ln in r0.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0
    assert rec["extrapolated"] is True and rec["cpu_baseline"]["extrapolated"] is True


def test_workloads_group_layers_by_input():
    sys.path.insert(0, ROOT)
    import bench
    block = bench.workload_layers("block_7b", bits=3)
    assert [len(g) for g in block] == [3, 1, 2, 1]          # qkv, o, gate/up, down
    assert all(s.bits == 3 and s.group == 128 for g in block for s in g)
    assert len({s.x_seed for s in block[0]}) == 1
    w = bench.work_model(block)
    assert w["weights"] == 4 * 4096 * 4096 + 2 * 11008 * 4096 + 4096 * 11008
    mlp = bench.workload_layers("mlp_65b", rank=1)
    assert [len(g) for g in mlp] == [2, 1]
    assert mlp[0][0].w_seed == 1 and mlp[0][0].x_seed == 101   # rank 1's own seeds
    down = bench.workload_layers("down_proj_65b")
    assert [(s.d_row, s.d_col, s.n_tokens, s.group) for g in down for s in g] == \
        [(8192, 22016, 131072, 128)]


def test_work_model_counts_each_route_work():
    """The prepare stage's fp64 work per input: 2/3 d^3 on the inverse route
    (Cholesky d^3/3 and triangular inverse d^3/3), d^3/3 + 128 d^2 on the
    factor route (the Cholesky and the panels V_ab G_bb); the other stages
    are the same on both."""
    sys.path.insert(0, ROOT)
    import bench
    mlp = bench.workload_layers("mlp_65b")           # inputs of d = 8192 and 22016
    inv = bench.work_model(mlp, "inverse")
    fac = bench.work_model(mlp, "factor")
    ds = [8192.0, 22016.0]
    assert inv["chol_flops"] == pytest.approx(sum(2 * d ** 3 / 3 for d in ds))
    assert fac["chol_flops"] == pytest.approx(sum(d ** 3 / 3 + 128 * d ** 2 for d in ds))
    for k in ("weights", "syrk_flops", "prop_flops", "pack_bytes"):
        assert inv[k] == fac[k]
    assert bench.work_model(mlp) == inv                 # the model's default argument
