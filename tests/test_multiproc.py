"""The N > 1 host path of bench.py on CPU with the gloo backend (world size 2): the only
cross-rank step is the max of the per-rank timings (measurement, not data path); the
reference arm runs on rank 0 only; the whole-job throughput counts every rank's batch."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks(1.0 + 2.5 * rank, torch.device("cpu"))
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"max": got}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        got = json.load(open(tmp_path / f"rank{r}.json"))["max"]
        assert got == pytest.approx(3.5)


def test_max_over_ranks_without_group_is_identity():
    assert bench.max_over_ranks(4.25) == 4.25


def test_weak_scaling_counts_every_rank():
    b = bench.algorithmic_bytes(8192, 2048, 4, 32)
    assert b == 42_991_616
    one = bench.job_throughput_gbs(b, 100, 1, 2.0)
    assert bench.job_throughput_gbs(b, 100, 2, 2.0) == pytest.approx(2 * one)


def test_reference_arm_runs_on_rank0_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
