"""The benchmark's clock record (CPU): samples come from an nvidia-smi log with host timestamps;
only those inside the timed region (give or take 20 ms of sampling jitter) count, throttle
reasons are collected from them, and a region too short for any sample falls back to the
nearest samples and says so."""
import datetime
import time

import bench


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        pass


def _log(path, t0, rows):
    """rows: (seconds after t0, sm MHz, sw_power_cap active?)"""
    with open(path, "w") as f:
        for dt, mhz, cap in rows:
            stamp = datetime.datetime.fromtimestamp(t0 + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
            f.write(f"{stamp}, 0, {mhz}, 1965, 700.00 W, 0x0000000000000000, Not Active, Not Active, "
                    f"Not Active, {'Active' if cap else 'Not Active'}\n")


def _sampler(t0, rows, begin, end):
    c = bench.ClockSampler(0)
    _log(c.path, t0, rows)
    c.proc, c.fh = _Done(), open(c.path, "a")
    c.t0, c.t1 = t0 + begin, t0 + end
    return c


def test_only_samples_inside_the_timed_region_count():
    t0 = time.time()
    rows = [(0.00, 345, True), (0.10, 1965, False), (0.12, 1965, True), (0.14, 1950, False),
            (0.16, 1965, False), (0.40, 600, True)]  # the first and last samples lie outside
    rec = _sampler(t0, rows, 0.095, 0.17).stop()
    assert rec["window"] == "timed region"
    assert rec["samples"] == 4
    assert rec["sm_mhz"] == 1965.0 and rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]


def test_short_region_reports_the_nearest_samples():
    """Only the two samples closest in time to the region stand in for it; idle samples further
    away (here a low-clock one with a throttle reason) are left out."""
    t0 = time.time()
    rows = [(0.0, 300, True), (0.15, 1965, False), (0.26, 1950, False), (0.9, 345, True)]
    rec = _sampler(t0, rows, 0.2, 0.21).stop()
    assert rec["window"] == "nearest samples to the timed region"
    assert rec["samples"] == 2
    assert rec["sm_mhz"] == 1957.5 and rec["reasons"] == []


def test_no_nvidia_smi_gives_no_record():
    c = bench.ClockSampler(0)
    c.proc = None
    assert c.stop() is None
