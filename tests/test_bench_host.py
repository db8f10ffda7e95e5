"""Host-side logic of bench.py, on CPU: the clock sampler against a fake
NVML (samples taken inside the timed region; a region shorter than one NVML
round trip gets the first sample after it; throttle reasons decoded from the
event-reason bits), and the name of the kernel the grouped GEMM launches
(the launch rule of fp4_gemm_grouped).  No GPU is used and no GPU setting
is read or changed."""
import os
import sys
import time
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture
def bench_with_fake_nvml(monkeypatch):
    fake = types.ModuleType("pynvml")
    fake.NVML_CLOCK_SM = 1
    fake.nvmlInit = lambda: None
    fake.nvmlDeviceGetHandleByPciBusId = lambda bus: 0
    fake.nvmlDeviceGetHandleByIndex = lambda i: 0
    fake.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        time.sleep(0.002)      # an NVML round trip
        return 1605

    fake.nvmlDeviceGetClockInfo = clock
    fake.nvmlDeviceGetCurrentClocksEventReasons = lambda h: 0x4   # sw_power_cap
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    sys.path.insert(0, ROOT)
    import bench
    import torch
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda d: (_ for _ in ()).throw(RuntimeError("no GPU")))
    return bench


def test_clocks_inside_region(bench_with_fake_nvml):
    c = bench_with_fake_nvml.Clocks(0)
    c.start()
    time.sleep(0.02)
    out = c.stop()
    assert out["source"] == "nvml 1 ms"
    assert out["samples"] >= 2
    assert out["sm_mhz"] == 1605.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_clocks_region_shorter_than_a_sample(bench_with_fake_nvml):
    c = bench_with_fake_nvml.Clocks(0)
    c.start()
    out = c.stop()
    assert out["samples"] >= 1
    assert out["sm_mhz"] == 1605.0


def test_grouped_kernel_name_follows_the_launch_rule():
    sys.path.insert(0, ROOT)
    import bench
    # groups averaging >= 512 rows with enough 256 x 256 tiles: CTA pairs
    assert "gemm_pair_kernel" in bench.grouped_kernel_name(16384, 4096, 8)
    # smaller groups: 128-row tiles, 256 wide unless N <= 128
    assert "128x256" in bench.grouped_kernel_name(16384, 2048, 64)
    assert "128x128" in bench.grouped_kernel_name(16384, 128, 8)
    assert "128x256" in bench.grouped_kernel_name(16384, 384, 256)   # any E up to 256
    # too few pair tiles for half the SMs: 128-row tiles
    assert "gemm_kernel" in bench.grouped_kernel_name(1024, 256, 1)
