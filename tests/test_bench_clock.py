"""bench.py's NVML clock sampler (host logic, no GPU): it reads the SM clock and
the clock-event reasons in a child process and keeps the samples taken inside
the timed region.  A fake NVML module stands in for the driver's library."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

FAKE_NVML = '''
NVML_CLOCK_SM = 1
def nvmlInit():
    if {fail}:
        raise RuntimeError("no NVML here")
def nvmlDeviceGetHandleByUUID(u): return 7
def nvmlDeviceGetHandleByIndex(i): return 7
def nvmlDeviceGetMaxClockInfo(h, c): return 1965
def nvmlDeviceGetClockInfo(h, c): return 1800
def nvmlDeviceGetCurrentClocksEventReasons(h): return 0x4 | 0x1   # sw_power_cap, gpu_idle
'''


def _sampler(tmp_path, monkeypatch, fail=False):
    (tmp_path / "pynvml.py").write_text(FAKE_NVML.format(fail=fail))
    monkeypatch.setenv("PYTHONPATH", str(tmp_path) + os.pathsep + os.environ.get("PYTHONPATH", ""))
    sys.path.insert(0, ROOT)
    try:
        import bench
    finally:
        sys.path.remove(ROOT)
    return bench.ClockSampler(0, period_s=0.002)


def test_samples_inside_the_region(tmp_path, monkeypatch):
    clk = _sampler(tmp_path, monkeypatch)
    with clk:
        time.sleep(0.3)
    s = clk.summary()
    assert clk.error is None
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] == 1800
    assert s["reasons"] == ["sw_power_cap"]   # gpu_idle is not reported
    # one sample per period at most (reads are instant here), and plenty of them
    assert 20 <= s["samples"] <= 0.3 / 0.002 + 5


def test_samples_after_the_region_are_dropped(tmp_path, monkeypatch):
    clk = _sampler(tmp_path, monkeypatch)
    with clk:
        pass   # an empty region: the child keeps sampling until told to stop
    assert clk.summary()["samples"] <= 2


def test_without_nvml_the_record_is_empty(tmp_path, monkeypatch):
    clk = _sampler(tmp_path, monkeypatch, fail=True)
    with clk:
        time.sleep(0.05)
    s = clk.summary()
    assert clk.error
    assert s == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
