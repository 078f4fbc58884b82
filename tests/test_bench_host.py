"""bench.py's multi-process plumbing on the CPU: two gloo ranks, each a
replica with its own timing, agree on the max time and the whole-job value;
the reference arm prints nothing on ranks other than 0."""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    ws, r, local = bench.dist_setup(backend="gloo")
    try:
        my_ms = 2.0 + 3.0 * r            # rank 1 is the slow replica
        bench.barrier(ws)
        ms = bench.max_over_ranks(my_ms, ws)
        out[r] = (ws, ms, bench.job_tflops(ws, 1e12, ms))
        bench.barrier(ws)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_replicas_take_the_max_time():
    world = 2
    out = mp.get_context("spawn").Manager().dict()  # no fork of this (threaded) process
    mp.spawn(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True)
    assert sorted(out.keys()) == [0, 1]
    for r in range(world):
        ws, ms, tflops = out[r]
        assert ws == 2 and ms == 5.0
        assert tflops == pytest.approx(2 * 1e12 / 5e-3 / 1e12)


def test_single_process_needs_no_process_group(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_setup(backend="gloo") == (1, 0, 0)
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.job_tflops(1, 2e12, 4.0) == pytest.approx(500.0)


def test_reference_arm_is_silent_off_rank_zero(monkeypatch):
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")

    class Args:
        steps, warmup = 1, 0

    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(Args())
    assert buf.getvalue() == ""


class _FakeNvml:
    """Stands in for the NVML binding: a fixed clock, power cap active on the 2nd reading."""
    NVML_CLOCK_SM = 1

    def __init__(self):
        self.calls = 0

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return 1900

    def nvmlDeviceGetCurrentClocksThrottleReasons(self, h):
        self.calls += 1
        return 0x4 if self.calls == 2 else 0


def test_clock_sampler_polls_nvml_during_the_region(monkeypatch):
    fake = _FakeNvml()
    monkeypatch.setattr(bench.Clocks, "_nvml_handle", lambda self: (fake, object()))
    with bench.Clocks(0, period_s=0.001) as clk:
        import time
        time.sleep(0.05)
    s = clk.summary()
    assert s["source"] == "nvml" and s["samples"] >= 3
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"]


def test_clock_sampler_parses_nvidia_smi_lines():
    clk = bench.Clocks(0)
    clk.proc = type("P", (), {"stdout": io.StringIO(
        "1965, 1965, Not Active, Not Active, Not Active, Not Active\n"
        "1800, 1965, Not Active, Active, Not Active, Active\n"
        "garbage\n")})()
    clk._read()
    s = clk.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1882.5 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
