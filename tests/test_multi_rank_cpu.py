"""Multi-process host logic of bench.py on CPU (gloo, world size 2).

The STA path shards by (batch, head) with no data exchange, so the only
cross-rank logic is the timing reduction (max over ranks) and the whole-job
throughput of weak scaling; the reference arm runs on rank 0 only.
"""
import datetime
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, queue):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(dist, 10.0 + rank, torch.device("cpu"))
        value = bench.weak_scaling_tflops(world, 1.0e12, ms)
        dist.barrier()
        queue.put((rank, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_max_time_and_sum_the_work():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(queue.get(timeout=10) for _ in range(2))
    for rank, ms, value in got:
        assert ms == 11.0
        assert value == pytest.approx(2 * 1.0e12 / 0.011 / 1e12)


def test_reference_arm_exits_quietly_on_other_ranks():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True,
                       timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_clock_records_that_are_measured_again():
    import bench
    cap = {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "samples": 10, "reasons": ["sw_power_cap"]}
    assert not bench.clocks_rejected(cap)  # the power cap alone is kept
    assert not bench.clocks_rejected(None)
    assert not bench.clocks_rejected({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "samples": 5, "reasons": []})
    for bad in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert bench.clocks_rejected({"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "samples": 5,
                                      "reasons": ["sw_power_cap", bad]})
    # clocks far below their maximum with no reason: a clock lock left behind
    assert bench.clocks_rejected({"sm_mhz": 1000.0, "sm_max_mhz": 1965.0, "samples": 5, "reasons": []})


def test_clock_record_covers_only_the_timed_region(monkeypatch):
    """The NVML sampler keeps only the samples taken between begin() and end()
    (a fake NVML stands in for the driver: idle clocks outside the region,
    power-capped clocks inside it)."""
    import time
    import types
    import bench
    inside = {"on": False}
    fake = types.ModuleType("pynvml")
    fake.NVML_CLOCK_SM = 1
    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByUUID = lambda u: "gpu"
    fake.nvmlDeviceGetHandleByIndex = lambda i: "gpu"
    fake.nvmlDeviceGetClockInfo = lambda h, c: 1575 if inside["on"] else 1965
    fake.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    fake.nvmlDeviceGetPowerUsage = lambda h: 990000 if inside["on"] else 150000
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4 if inside["on"] else 0x1
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: types.SimpleNamespace(uuid="fake"))
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.1)  # idle samples before the region
    inside["on"] = True
    s.begin()
    time.sleep(0.2)
    s.end()
    inside["on"] = False
    time.sleep(0.1)  # idle samples after it
    rec = s.stop()
    assert rec["window"] == "timed region" and rec["samples"] >= 3
    assert rec["sm_mhz"] == 1575.0 and rec["sm_max_mhz"] == 1965.0 and rec["power_w"] == 990.0
    assert rec["reasons"] == ["sw_power_cap"] and not rec["rejected"]
