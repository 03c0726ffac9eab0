"""Host-side logic of bench.py on the CPU: the multi-rank reductions run as
two gloo ranks, per-rank batches differ, the FLOP count matches its closed
form, and the reference arm (the oracle on the host cores) prints a valid
line."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch
    dist = bench.init_dist(world, "gloo")
    mx = bench.reduce_max(1.5 + rank, dist, torch.device("cpu"))
    sm = bench.reduce_sum(10.0 * (rank + 1), dist, torch.device("cpu"))
    q.put((rank, mx, sm, bench.rank_seed(rank), bench.dist_env()))
    dist.destroy_process_group()


def test_two_rank_reductions():
    import torch.multiprocessing as mp
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
    assert [r[1] for r in res] == [2.5, 2.5]
    assert [r[2] for r in res] == [30.0, 30.0]
    assert res[0][3] != res[1][3]
    assert res[1][4] == (1, 2, 1)


def test_flops_closed_form():
    assert bench.so2_flops_per_edge(4, 128) == 4751360
    assert bench.so2_flops_per_edge(6, 128) == 13533184
    assert bench.so2_flops_per_edge(2, 8) == 3712


def test_rank_batches_differ():
    from atomistic_mlip_b200 import workloads as w
    a = w.make_workload(1, seed=bench.rank_seed(0), C=8, L=1, H=1)
    b = w.make_workload(1, seed=bench.rank_seed(1), C=8, L=1, H=1)
    assert a.N != b.N or not np.array_equal(a.pos, b.pos)


def test_reference_arm_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, env=env, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "edges/s"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2"],
                         capture_output=True, text=True, env=env, timeout=120, cwd=ROOT)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_gpus_flag_must_match_world_size():
    """--gpus N without N ranks fails loudly instead of measuring one GPU."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--gpus", "8"],
                         capture_output=True, text=True, env=env, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "WORLD_SIZE" in out.stderr


def test_linear_fit():
    fit = bench.linear_fit([10, 30, 100], [1000 + 40 * n for n in (10, 30, 100)])
    assert abs(fit["bytes_per_atom"] - 40) < 1e-9 and abs(fit["intercept_bytes"] - 1000) < 1e-6
    assert abs(fit["r2"] - 1.0) < 1e-12
