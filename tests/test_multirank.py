"""The N>1 path of the bench: replicas, one per rank, with no collective on
the data path.  The process group only carries barriers and the max-over-ranks
timing reduction; these tests run it on two `gloo` ranks on the CPU and check
what rank 0 reports and that the other ranks of the reference arm exit without
work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist = bench.init_group(world, backend="gloo")
    # each rank's own step time; the job is as slow as its slowest replica
    ms = 1.0 + 0.5 * rank
    job_ms = bench.max_over_ranks(ms, dist)
    dist.barrier()
    out.put((rank, job_ms, bench.job_rate(1, world, job_ms)))
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_max_over_ranks_gloo(world):
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    slowest = 1.0 + 0.5 * (world - 1)
    for r, job_ms, rate in res:
        assert job_ms == slowest
        assert rate == pytest.approx(world * 1e3 / slowest)


def test_single_rank_has_no_group():
    assert bench.init_group(1) is None
    assert bench.max_over_ranks(3.25, None) == 3.25
    assert bench.job_rate(1, 1, 2.0) == 500.0


def _run_bench(rank, world, *extra):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus",
                           str(world), "--steps", "1", "--warmup", "0", *extra],
                          env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)


@pytest.mark.parametrize("workload", ["decode-64k", "eval-window"])
def test_reference_arm_other_ranks_exit_without_work(workload):
    r = _run_bench(1, 2, "--workload", workload)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_arm_rank0_line():
    r = _run_bench(0, 2)
    assert r.returncode == 0, r.stderr
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference"
    assert line["n_gpus"] == 2 and line["scaling"] == "weak"
    assert line["config"]["parallelism"] == "replicas x2"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
