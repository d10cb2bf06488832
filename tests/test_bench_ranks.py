"""Multi-rank host logic of bench.py on CPU: two gloo ranks (replicas), max over ranks,
whole-job value, and the reference arm running on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    sys.path.insert(0, ROOT)
    import bench
    vals = bench.max_over_ranks([10.0 + rank, 5.0 - rank, 7.0], world)
    dist.destroy_process_group()
    q.put((rank, vals))


def test_max_over_ranks_gloo_world2():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0] == out[1] == [11.0, 5.0, 7.0]


def test_job_value_is_per_call_over_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_us_per_call(100.0, 50, 1) == pytest.approx(2000.0)
    assert bench.job_us_per_call(100.0, 50, 4) == pytest.approx(500.0)


def test_reference_arm_non_zero_rank_exits_without_output():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "1", "--warmup", "0"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_reference_arm_rank0_prints_contract_line():
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--workload", "tiny", "--steps", "2", "--warmup", "3"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["steps"] == 2 and line["unit"] == "us/call"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["higher_is_better"] is False and line["value"] > 0


def test_tensor_peak_follows_the_clock_record():
    # burst cuBLAS figure while the SM clock stays near its maximum; the sustained
    # (power-capped) figure only when the record shows the clock pulled down by the cap
    sys.path.insert(0, ROOT)
    import bench
    burst, sust = 1642.8, 1402.8
    assert bench.tensor_peak({"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}, burst, sust, "m")[0] == burst
    assert bench.tensor_peak({"sm_mhz": 1916.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}, burst, sust,
                             "m")[0] == burst
    assert bench.tensor_peak({"sm_mhz": 1620.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}, burst, sust,
                             "m")[0] == sust
    # a low clock with no power-cap reason is not power capping: burst, and the run is
    # flagged by its clock record instead
    assert bench.tensor_peak({"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": []}, burst, sust, "m")[0] == burst
    assert bench.tensor_peak({"sm_mhz": None, "sm_max_mhz": None, "reasons": []}, burst, sust, "m")[0] == burst


def test_exchange_workloads_have_no_oracle_arm():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload",
                        "tp8_reduce"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0
    import json
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and "unavailable" in line
