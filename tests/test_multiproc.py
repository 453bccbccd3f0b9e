"""The N>1 path of bench.py on CPU: world-size-2 gloo ranks (replicas, no data-path
collective; the job time is the max over ranks, and rank 0 alone reports)."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [12.5, 40.0][rank]                      # rank 1 is the slow one
        mx = bench.reduce_max(ms, world, "cpu")
        val = bench.job_tokens_per_s(world, 4096, 10, mx)
        q.put((rank, mx, val))
    finally:
        torch.distributed.destroy_process_group()


def test_reduce_max_and_job_throughput_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(2))
    for rank, mx, val in got:
        assert mx == 40.0                            # every rank sees the slowest rank's time
        assert val == pytest.approx(2 * 4096 * 10 / 0.040)


def test_reference_arm_only_rank0_runs():
    # a rank other than 0 exits 0 without work and prints nothing
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_gpus_must_match_the_launched_world():
    # a world of 2 ranks launched for --gpus 4 (or --gpus left at 1) is refused, not mislabelled
    for gpus in ("4", "1"):
        env = dict(os.environ, RANK="0", WORLD_SIZE="2", LOCAL_RANK="0")
        r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                            "tiny", "--gpus", gpus, "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                           text=True, timeout=300)
        assert r.returncode == 2 and r.stdout.strip() == "" and "WORLD_SIZE=2" in r.stderr


def test_reference_arm_rank0_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                        "--steps", "2", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    import json
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["e2e"]["h2d_bytes_per_step"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle"
