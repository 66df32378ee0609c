"""bench.py's clock sampler keeps the nvidia-smi samples stamped inside the
timed region (host logic only: the nvidia-smi process is replaced by a fake
and its output by canned lines)."""

import datetime
import importlib.util
import os
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


class _FakeProc:
    def terminate(self):
        pass

    def kill(self):
        pass

    def wait(self, timeout=None):
        return 0


def _stamp(t):
    return datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]


def _sampler(lines):
    b = _bench()
    s = b.ClockSampler.__new__(b.ClockSampler)
    s.proc = _FakeProc()
    s.reader = None
    s.lines = [line + "\n" for line in lines]
    return s


def test_samples_inside_the_region_only():
    t = time.time()
    lines = [f"{_stamp(t + 0.02 * k)}, 0, {1965 - 10 * k}, 1965, 900.0, 0x4, Not Active, Not Active, "
             f"Not Active, {'Active' if k >= 8 else 'Not Active'}" for k in range(10)]
    c = _sampler(lines).stop(t + 0.05, t + 0.15)
    # samples k = 3..7 lie inside; their clocks are 1935..1895, median 1915
    assert c["samples"] == 5
    assert c["sm_mhz"] == 1915.0
    assert c["reasons"] == []  # sw_power_cap only outside the region
    assert c["window"] == "timed region"


def test_falls_back_to_all_samples_when_none_inside():
    t = time.time()
    lines = [f"{_stamp(t + 0.02 * k)}, 0, 1800, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active"
             for k in range(4)]
    c = _sampler(lines).stop(t + 10, t + 11)
    assert c["samples"] == 4
    assert c["reasons"] == ["sw_power_cap"]
    assert c["window"].startswith("whole sampling period")


def test_malformed_lines_are_skipped():
    t = time.time()
    lines = ["garbage", "", f"{_stamp(t + 0.01)}, 0, 1965, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, "
             "Not Active", "[N/A], 0, x, y"]
    c = _sampler(lines).stop(t, t + 1)
    assert c["samples"] == 1 and c["sm_mhz"] == 1965.0


def test_wait_ready_returns_once_a_sample_arrived():
    t = time.time()
    s = _sampler([f"{_stamp(t)}, 0, 1965, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Not Active"])
    assert s.wait_ready(timeout=0.1) is True


def test_wait_ready_gives_up_after_its_timeout():
    s = _sampler([])
    t = time.time()
    assert s.wait_ready(timeout=0.1) is False
    assert time.time() - t < 1.0
