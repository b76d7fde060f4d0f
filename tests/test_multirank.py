"""The multi-rank benchmark path on the CPU (gloo, world size 2).

The layer partitions over tokens: every rank runs its own batch with
replicated weights and no data-path collective; the only cross-rank
operations are the timing reduction (max of the step time, sum of the work)
and, for the reference arm, that only rank 0 runs and prints.
"""
import argparse
import os
import socket
import tempfile

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from rotated_w4a4_quantized_b200 import workloads as wl


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _aggregate_rank(rank: int, world: int, port: int, out_dir: str):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms, ops = bench.aggregate(1.5 + rank, 10.0 * (rank + 1))
        with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
            f.write(f"{ms} {ops}\n")
    finally:
        dist.destroy_process_group()


def test_aggregate_takes_max_time_and_total_work_over_two_ranks():
    port = _free_port()
    with tempfile.TemporaryDirectory() as d:
        mp.start_processes(_aggregate_rank, args=(2, port, d), nprocs=2, join=True,
                           start_method="spawn")
        for rank in range(2):
            with open(os.path.join(d, f"rank{rank}.txt")) as f:
                ms, ops = map(float, f.read().split())
            assert ms == 2.5            # the slowest rank's time
            assert ops == 30.0          # every rank's work


def test_aggregate_is_local_without_a_process_group():
    assert not dist.is_initialized()
    assert bench.aggregate(3.25, 7.0) == (3.25, 7.0)


def test_each_rank_runs_its_own_batch_of_the_same_shape():
    name = "small_g256"
    seed = wl.WORKLOADS[name].seed
    r0 = wl.make_workload(name, seed=seed + 0)
    r1 = wl.make_workload(name, seed=seed + 1)
    assert [l.spec for l in r0] == [l.spec for l in r1]
    for a, b in zip(r0, r1):
        assert a.x.shape == b.x.shape and a.w.shape == b.w.shape
        assert not torch.equal(a.x, b.x)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = argparse.Namespace(workload="small_g256", steps=3, warmup=3, cpu_seconds=0.1,
                              variant="w4a4")
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""


def test_w4a16_reference_arm_runs_on_rank_zero_only(monkeypatch, capsys):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("LOCAL_RANK", "1")
    args = argparse.Namespace(workload="small_g256", steps=3, warmup=3, cpu_seconds=0.1,
                              variant="w4a16")
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""


def test_w4a16_reference_arm_line(monkeypatch, capsys):
    import json
    for v in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(v, raising=False)
    args = argparse.Namespace(workload="small_g256", steps=3, warmup=3, cpu_seconds=0.1,
                              variant="w4a16")
    bench.run_reference(args)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "TFLOP/s" and line["dtype"] == "bf16"
    assert line["metric"] == bench.METRIC_W4A16 and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_hash_covers_the_w4a4_library_sources():
    """The per-launch DRAM traffic the benchmark reports belongs to the W4A4
    kernels; its key hashes exactly the files that library is built from."""
    from rotated_w4a4_quantized_b200 import build
    assert sorted(os.path.basename(p) for p in build.DEPS) == sorted(bench.W4A4_SOURCES)


def test_rank_plan_spawns_runs_or_refuses():
    import pytest
    assert bench.rank_plan(1, {}) == "run"
    assert bench.rank_plan(4, {}) == "spawn"
    assert bench.rank_plan(2, {"WORLD_SIZE": "2"}) == "run"
    assert bench.rank_plan(1, {"WORLD_SIZE": "1"}) == "run"
    with pytest.raises(SystemExit):
        bench.rank_plan(8, {"WORLD_SIZE": "2"})      # a process group of another size
    with pytest.raises(SystemExit):
        bench.rank_plan(0, {})
    cmd = bench.spawn_cmd(4, ["--gpus", "4", "--steps", "7"], 29512)
    assert cmd[1:3] == ["-m", "torch.distributed.run"]
    assert "--nproc-per-node=4" in cmd and "127.0.0.1" in cmd and cmd[-4:] == [
        "--gpus", "4", "--steps", "7"]


def test_gpus_without_torchrun_launches_the_ranks_itself():
    """`bench.py --gpus 2` outside torchrun starts two ranks; the reference
    arm (the CPU oracle, no GPU needed) runs on rank 0 alone, which prints
    the only JSON line, with n_gpus = 2."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.abspath(bench.__file__))
    env = {k: v for k, v in os.environ.items()
           if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3", "--workload", "small_g256",
                        "--cpu-seconds", "0.2"], capture_output=True, text=True, timeout=600,
                       cwd=root, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2
