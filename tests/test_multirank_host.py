"""Multi-rank host logic of the benchmark, on CPU with the gloo backend
(world size 2): the path shards by independent layers (weak scaling), so the
only collective is the max over ranks of the step time.  Also the reference
arm's launch contract: under torchrun rank 0 alone prints one JSON line."""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import linear_problem  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # each rank's own step time; every rank must see the slowest one
        ms = bench.max_over_ranks(torch, dist, 1.5 + rank, "cpu")
        # each rank draws its own layer: gather a fingerprint of its input
        p = linear_problem(bench.rank_seed(1, rank), 0, 512, 64, 2, K=2)
        fp = torch.tensor([float(p.x.sum()), float(p.theta.sum())], dtype=torch.float64)
        allfp = [torch.zeros_like(fp) for _ in range(world)]
        dist.all_gather(allfp, fp)
        dist.barrier()
        q.put((rank, ms, [t.tolist() for t in allfp]))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_max_time_and_distinct_layers():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    assert [r[1] for r in res] == [2.5, 2.5]          # max over ranks, identical on both
    fps = res[0][2]
    assert res[1][2] == fps and fps[0] != fps[1]      # ranks hold different layers


def test_whole_job_rate_is_weak_scaling():
    # every rank moves the same bytes per step; the job's rate counts all ranks
    assert bench.whole_job_rate(1e9, 1, 1000.0) == pytest.approx(1e9)
    assert bench.whole_job_rate(1e9, 4, 1000.0) == pytest.approx(4e9)
    assert bench.whole_job_rate(1e9, 4, 2000.0) == pytest.approx(2e9)
    assert bench.max_over_ranks(None, None, 3.0, "cpu") == 3.0
    assert len({bench.rank_seed(1, r) for r in range(8)}) == 8


def _run_bench(args, env=None, timeout=300):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, "bench.py"] + args, cwd=ROOT, env=e, capture_output=True, text=True,
                          timeout=timeout)


def test_reference_arm_json_line():
    r = _run_bench(["--impl", "reference", "--config", "0", "--steps", "4", "--warmup", "3"])
    assert r.returncode == 0, r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["unit"] == "GB/s" and out["value"] > 0
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["value"] == out["value"]
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0
    assert out["steps"] == 4 and out["warmup"] == 3


def test_reference_arm_other_ranks_do_no_work():
    r = _run_bench(["--impl", "reference", "--config", "0", "--steps", "4", "--warmup", "3"],
                   env={"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_bounded_rows():
    # a long run samples fewer output rows per step (multiples of 16, at least 16)
    probs, sub_m, M = bench.oracle_problems(0, None)
    few = bench.reference_rows(probs, 3, 3, seconds=60.0)
    many = bench.reference_rows(probs, 10 ** 7, 3, seconds=1.0)
    assert few == [512] and many == [16]
    t, b = bench.oracle_run(probs, 0, many)
    assert b == bench.linear_bytes(512, 16, 4)


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--config", "0", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1 and json.loads(lines[0])["n_gpus"] == 2
