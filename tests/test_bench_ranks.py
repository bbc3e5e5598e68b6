"""The host side of bench.py's multi-GPU path on the CPU: two gloo ranks reduce their times to
the slowest one and the whole-job throughput counts every rank's tokens; the reference arm runs
on rank 0 alone and the other ranks leave without work."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, values, out_dir):
    import datetime

    import torch.distributed as dist

    sys.path.insert(0, ROOT)
    import bench

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.reduce_max(values[rank], dist)
        dist.barrier()
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"ms": ms, "tok_s": bench.job_tokens_per_s(world, 64, 10, ms)}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time(tmp_path):
    values = [1.5, 2.5]
    mp.spawn(_rank, args=(2, _free_port(), values, str(tmp_path)), nprocs=2, join=True)
    got = [json.load(open(tmp_path / f"r{r}.json")) for r in range(2)]
    assert [g["ms"] for g in got] == [2.5, 2.5]
    # 2 ranks x 64 tokens x 10 steps in 2.5 ms
    assert got[0]["tok_s"] == pytest.approx(2 * 64 * 10 / 2.5e-3)


def test_reduce_max_without_a_process_group_is_the_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25) == 3.25


def _run_reference(rank: int):
    env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank))
    return subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--gpus", "2",
                           "--steps", "1", "--warmup", "3"], cwd=ROOT, env=env, capture_output=True, text=True,
                          timeout=300)


def test_reference_arm_runs_on_rank_zero_only():
    r1 = _run_reference(1)
    assert r1.returncode == 0, r1.stderr
    assert r1.stdout.strip() == ""
    r0 = _run_reference(0)
    assert r0.returncode == 0, r0.stderr
    line = json.loads(r0.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
