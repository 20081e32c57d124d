"""bench.py's multi-rank plumbing on CPU: two gloo ranks, max-over-ranks timing,
whole-job throughput, and the reference arm running on rank 0 only."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ranks = bench.Ranks(world, device="cpu")
        ranks.barrier()
        # rank r ran 100 * (r + 1) units in 10 * (r + 1) ms
        rate, ms = bench.whole_job_rate(ranks, 100.0 * (rank + 1), 10.0 * (rank + 1))
        q.put((rank, rate, ms, ranks.max(rank), ranks.sum(1.0)))
        ranks.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_aggregate_as_the_slowest_rank():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, PORT, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, rate, ms, mx, sm in res:
        # units 100 + 200 over the slowest rank's 20 ms
        assert ms == pytest.approx(20.0)
        assert rate == pytest.approx(300.0 / 0.020)
        assert mx == 1 and sm == 2


PORT = _free_port()


def test_reference_arm_only_rank0_prints(tmp_path):
    """Under a 2-rank launch the reference arm's non-zero rank exits 0 without work."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_json_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "2",
                        "--warmup", "1", "--ref-seconds", "3"], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
