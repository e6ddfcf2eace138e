"""Multi-rank plumbing of bench.py on CPU: two gloo ranks, the reference arm
under torchrun-style environments.  No GPU is touched."""
import json
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


def _rank_worker(rank, world, port, out_dir):
    import datetime
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        bench.sync_ranks(world)
        # each rank "took" a different time; the job took the slowest one's
        total_ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        rate = bench.job_rate(world, 100, total_ms)
        bench.sync_ranks(world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"total_ms": total_ms, "rate": rate}, f)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_agree_on_max_and_job_rate(tmp_path):
    world = 2
    mp.start_processes(_rank_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["total_ms"] == 15.0          # the slower rank's time, on every rank
        assert g["rate"] == pytest.approx(world * 100 / 0.015)


def test_single_process_helpers_need_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    bench.sync_ranks(1)
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.job_rate(1, 10, 20.0) == pytest.approx(500.0)


def test_reference_arm_on_a_nonzero_rank_prints_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1",
               MASTER_ADDR="127.0.0.1", MASTER_PORT=str(_free_port()))
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


def test_reference_line_shape(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    def fake_baseline(st, host=None):
        return {"value": None, "unit": "step/s", "cores": 4, "kind": "oracle",
                "sample": "stub", "s_per_step": 2.0}

    monkeypatch.setattr(bench, "cpu_baseline", fake_baseline)
    monkeypatch.setattr(bench.inputs, "make", lambda name: None)

    class A:
        steps_ref = 2
        warmup_ref = 0

    assert bench.run_reference(A(), rank=1) is None
    line = bench.run_reference(A(), rank=0)
    assert line["impl"] == "reference"
    assert line["value"] == pytest.approx(0.5)
    assert line["unit"] == "step/s" and line["higher_is_better"] is True
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "step/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_runs_the_gpu_arms_step_counts():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reference_plan(20, 5) == (20, 5)      # the driver's K and W: exactly those
    assert bench.reference_plan(3, 3) == (3, 3)
    timed, untimed = bench.reference_plan(2000, 20)   # the default K would take hours
    assert 1 <= timed and timed + untimed <= bench.REF_BUDGET_S // bench.REF_STEP_S_EST
