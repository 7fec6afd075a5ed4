"""Host logic of bench.py under several ranks (gloo on the CPU, world size 2): the
step time is the maximum over ranks and the throughput counts the work of every rank.
The reference arm prints from rank 0 only."""

import json
import os
import socket
import subprocess
import sys

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime

    import bench
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks([10.0 + rank, 5.0 - rank], "cpu")
        out[rank] = got
    finally:
        torch.distributed.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    for r in range(world):
        assert res[r] == [11.0, 5.0]


def test_whole_job_throughput_counts_all_ranks():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.whole_job_tflops(2.0e12, 1, 4.0)
    assert abs(one - 500.0) < 1e-9
    assert abs(bench.whole_job_tflops(2.0e12, 8, 4.0) - 8 * one) < 1e-6


def test_reference_arm_prints_on_rank0_only():
    """Non-zero ranks of the reference arm exit 0 without output (the oracle runs on
    rank 0 only)."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_line_rank0_small():
    """Rank 0 prints one JSON line with the contract keys (tiny workload to stay fast)."""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for k in ("impl", "metric", "value", "unit", "cpu_baseline", "e2e", "higher_is_better"):
        assert k in line
    assert line["impl"] == "reference" and line["value"] > 0


def test_applicable_peak_burst_for_short_regions():
    """A timed region under a second is held to the burst peak, a longer one to the
    sustained (power-capped) peak; the label says which."""
    sys.path.insert(0, ROOT)
    import bench
    peaks = {"bf16_tflops": 1683.8, "bf16_tflops_sustained": 1391.3}
    p, why = bench.applicable_peak(peaks, "measured", 0.074)
    assert p == 1683.8 and "burst" in why
    p, why = bench.applicable_peak(peaks, "measured", 1.5)
    assert p == 1391.3 and "sustained" in why


def test_clock_record_of_a_region_shorter_than_the_period():
    """No sample falls inside a 20 ms region between two samples: the record keeps the
    nearest sample on each side instead of reporting none; reasons are unioned."""
    sys.path.insert(0, ROOT)
    import bench
    cs = bench.ClockSampler(0)
    cs.source = "nvml"
    cs.samples = [(10.00, 1965.0, 1965.0, set()), (10.10, 1950.0, 1965.0, {"sw_power_cap"}),
                  (10.20, 1965.0, 1965.0, set())]
    cs.t_begin, cs.t_end = 10.12, 10.14
    r = cs.stop()
    assert r["samples"] == 2 and r["sm_mhz"] == (1950.0 + 1965.0) / 2 and r["reasons"] == ["sw_power_cap"]
    assert "nearest" in r["kept"]
    cs.samples.append((10.13, 1900.0, 1965.0, set()))
    r = cs.stop()
    assert r["samples"] == 1 and r["sm_mhz"] == 1900.0 and r["kept"] == "inside the timed region"
