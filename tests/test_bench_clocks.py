"""The benchmark's clock sampler on CPU, against a stand-in NVML module: the
polling runs in a child process, only samples stamped inside the sampled
region are kept, and a sampler that cannot start leaves a note, not a hang."""
import os
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

FAKE_NVML = '''
NVML_CLOCK_SM = 1
def nvmlInit():
    {init}
def nvmlDeviceGetHandleByUUID(u):
    assert u == "GPU-test"
    return u
def nvmlDeviceGetMaxClockInfo(h, c):
    return 1965
def nvmlDeviceGetClockInfo(h, c):
    return 1920
def nvmlDeviceGetCurrentClocksEventReasons(h):
    return 0x4 | 0x1
'''


def _fake(tmp_path, monkeypatch, init="pass"):
    (tmp_path / "pynvml.py").write_text(FAKE_NVML.format(init=init))
    monkeypatch.setenv("PYTHONPATH", str(tmp_path) + os.pathsep + os.environ.get("PYTHONPATH", ""))


def test_samples_inside_region(tmp_path, monkeypatch):
    import bench
    _fake(tmp_path, monkeypatch)
    t_before = time.monotonic()
    with bench.ClockSampler(0, uuid="GPU-test") as c:
        t_in = time.monotonic()
        time.sleep(0.05)
    assert c.err is None, c.err
    assert c.proc is None            # the child has exited
    assert c.t0 >= t_before and c.t0 <= t_in
    s = c.summary()
    assert s["sm_mhz"] == 1920 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]      # gpu_idle is not reported
    assert s["samples"] >= 5                     # 0.5 ms polling over 50 ms


def test_short_region_keeps_nearest_sample(tmp_path, monkeypatch):
    import bench
    _fake(tmp_path, monkeypatch)
    with bench.ClockSampler(0, period_s=5.0, uuid="GPU-test") as c:
        pass
    assert c.err is None, c.err
    assert c.summary()["samples"] == 1


def test_sampler_that_cannot_start(tmp_path, monkeypatch):
    import bench
    _fake(tmp_path, monkeypatch, init="raise RuntimeError('no driver')")
    t = time.monotonic()
    with bench.ClockSampler(0, uuid="GPU-test") as c:
        pass
    assert time.monotonic() - t < 30
    s = c.summary()
    assert s["samples"] == 0 and s["sm_mhz"] is None
    assert "no driver" in s["note"]


def test_mark_drops_earlier_samples(tmp_path, monkeypatch):
    import bench
    _fake(tmp_path, monkeypatch)
    c = bench.ClockSampler(0, period_s=0.001, uuid="GPU-test").start()
    time.sleep(0.2)                  # about 200 samples before the mark
    c.mark()
    time.sleep(0.02)
    c.stop()
    assert c.err is None, c.err
    assert 1 <= c.summary()["samples"] <= 60
