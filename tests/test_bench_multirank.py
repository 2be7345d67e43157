"""The benchmark's multi-rank host logic on CPU: two gloo ranks gather their
timing records and rank 0 forms the whole-job figures (weak scaling: bytes of
all ranks over the slowest rank's time); the reference arm runs on rank 0
only and prints one JSON line."""
import datetime
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


def _worker(rank, world, port, results):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local = {"ms": 100.0 + 10.0 * rank, "bytes": 1e9 * (rank + 1), "e2e_ms": 50.0 + rank,
                 "e2e_bytes": 2e8}
        per = bench.gather_rank_stats(local, world)
        results[rank] = bench.combine_rank_stats(per, steps=4)
    finally:
        dist.destroy_process_group()


def test_two_ranks_gather_and_combine():
    world = 2
    with mp.get_context("spawn").Manager() as mgr:
        results = mgr.dict()
        mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(results)
    assert set(res) == {0, 1}
    for r in res.values():  # every rank sees the same whole-job figures
        assert r["ms_max"] == 110.0
        assert r["value"] == pytest.approx(3e9 / 0.110 / 1e9)
        assert r["ms_per_step"] == pytest.approx(27.5)
        assert r["e2e_value"] == pytest.approx(4e8 / 0.051 / 1e9)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_1k", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_prints_one_line():
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_1k", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    # the same `config` object as the CUDA arm prints for this workload, and the time of what it ran
    sys.path.insert(0, ROOT)
    import bench
    from long_context_decoding_saga_b200 import workload
    assert line["config"] == bench.workload_config(workload.by_name("tiny_1k"), 1)
    assert line["timed_unit"] == "one layer-step (layer 0)"
