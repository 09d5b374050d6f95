"""Host-side logic of the multi-process bench, on the CPU: the replicated step is timed as
the slowest rank's time (max over ranks through the process group, here gloo with two
ranks), the whole-job value counts every rank's units, and the reference arm runs on rank 0
only (the other ranks exit 0 without work)."""

import os
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, out_path):
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(local_ms, torch.device("cpu"))
        value = bench.job_value(1e9, world, ms)
        with open(f"{out_path}.{rank}", "w") as f:
            f.write(f"{ms} {value}")
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo(tmp_path):
    world = 2
    port = 29500 + os.getpid() % 1000
    out = str(tmp_path / "r")
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    for r in range(world):
        ms, value = map(float, open(f"{out}.{r}").read().split())
        assert ms == 5.0  # every rank sees the slowest rank's time
        # 2 ranks x 1e9 bytes in 5 ms = 400 GB/s for the whole job
        assert value == pytest.approx(2 * 1e9 / 5e-3 / 1e9)


def test_max_over_ranks_single_process():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.5, torch.device("cpu")) == 7.5
    assert bench.job_value(2e9, 1, 2.0) == pytest.approx(1000.0)


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "1"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_detail_oracle_baselines_run_on_cpu():
    sys.path.insert(0, ROOT)
    import bench
    samples = bench.oracle_detail_samples(frac_rows=64)
    assert set(samples) == {"q4_0_decode_M1_step", "backward_x_M1_14336x4096"}
    for name, (run, nbytes, text) in samples.items():
        r = bench.time_oracle(run, nbytes, text, seconds=0.2)
        assert r["kind"] == "oracle" and r["value"] > 0 and nbytes > 0, name
    bad = bench.time_oracle(lambda: 1 / 0, 1, "x", seconds=0.1)
    assert bad["value"] is None and "error" in bad
