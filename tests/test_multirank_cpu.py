"""The N > 1 path of bench.py, on CPU ranks (gloo, world size 2).

Every rank decodes its own independent batch (replicas, weak scaling); the
only collectives are the max of the step times and the sum of the bytes each
rank processed.  These tests run that aggregation across two real gloo
processes, and the reference arm's rank handling (rank 0 alone runs and
prints; other ranks exit 0 without work).
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        red = bench.RankReducer(world, "cpu")
        # rank r: a step of (1 + r) ms over (r + 1) * 1e9 bytes
        step, total, value = bench.aggregate_step(1.0 + rank, (rank + 1) * 10**9, red)
        # a second round of calls in the same order on every rank
        extra = red.max(-float(rank)), red.sum(0.5)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"step": step, "total": total, "value": value, "extra": extra}, f)
    finally:
        dist.destroy_process_group()


def test_aggregate_over_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r in res:
        # slowest rank's time, every rank's bytes: whole-job throughput
        assert r["step"] == 2.0
        assert r["total"] == 3 * 10**9
        assert r["value"] == pytest.approx(3e9 / 2e-3 / 1e9)
        assert r["extra"] == [0.0, 1.0]


def test_aggregate_is_identity_on_one_rank():
    sys.path.insert(0, ROOT)
    import bench
    step, total, value = bench.aggregate_step(4.0, 8 * 10**9, bench.RankReducer(1))
    assert (step, total) == (4.0, 8 * 10**9)
    assert value == pytest.approx(8e9 / 4e-3 / 1e9)


def _run_reference(rank: int, world: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config",
                           "tiny", "--gpus", str(world), "--steps", "2", "--warmup", "1"],
                          env=env, capture_output=True, text=True, timeout=300, cwd=ROOT)


def test_reference_arm_runs_on_rank_zero_only():
    p1 = _run_reference(1, 2)
    assert p1.returncode == 0, p1.stderr
    assert p1.stdout.strip() == ""
    p0 = _run_reference(0, 2)
    assert p0.returncode == 0, p0.stderr
    lines = [l for l in p0.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"] and line["value"] > 0
