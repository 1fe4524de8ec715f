"""Host-side pieces of bench.py that need no GPU: the clock sampler keeps only
the nvidia-smi samples inside the timed region and reports throttle reasons."""

import os
import tempfile
import time
from datetime import datetime

import bench


def _sampler(rows, t0, t1):
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    for when, mhz, reasons in rows:
        stamp = datetime.fromtimestamp(when).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        flags = ["Active" if n in reasons else "Not Active"
                 for n in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")]
        c.f.write(f"{stamp}, 0, {mhz}, 1965, 700.0, 0x0, {', '.join(flags)}\n")
    c.f.flush()

    class _Proc:
        def terminate(self):
            pass

        def wait(self):
            pass

    c.p = _Proc()
    c.t0, c.t1 = t0, t1
    return c


def test_clock_samples_inside_the_timed_region_only():
    now = time.time()
    rows = [(now - 1.0, 1000, ()), (now + 0.1, 1800, ("sw_power_cap",)), (now + 0.3, 1900, ()),
            (now + 2.0, 1200, ("hw_slowdown",))]
    c = _sampler(rows, now, now + 0.5)
    name = c.f.name
    r = c.stop()
    assert r["samples"] == 2 and r["sm_mhz"] == 1850.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"] and r["window"] == "timed region"
    assert not os.path.exists(name)


def test_short_region_takes_the_first_sample_after_its_start():
    now = time.time()
    rows = [(now - 0.5, 1000, ()), (now + 0.08, 1700, ("hw_thermal_slowdown",))]
    r = _sampler(rows, now, now + 0.01).stop()
    assert r["samples"] == 1 and r["sm_mhz"] == 1700.0
    assert r["reasons"] == ["hw_thermal_slowdown"] and r["window"].startswith("first sample after")


def test_no_samples_gives_none():
    assert _sampler([], time.time(), time.time() + 1).stop() is None


def test_roofline_peak_matches_the_timed_region():
    import bench
    burst, sustained = 1674.3, 1409.4
    # A short region at full clock: the burst GEMM figure.
    p, kind = bench.roofline_peak(burst, sustained, 24.0, {"reasons": [], "sm_mhz": 1965.0})
    assert p == burst and kind.startswith("burst")
    # A short region that saw the power cap is still a burst measurement.
    assert bench.roofline_peak(burst, sustained, 300.0, {"reasons": ["sw_power_cap"]})[0] == burst
    # Only a region of a second or more under the power cap pairs with the sustained figure.
    p, kind = bench.roofline_peak(burst, sustained, 1300.0, {"reasons": ["sw_power_cap"]})
    assert p == sustained and kind.startswith("sustained")
    assert bench.roofline_peak(burst, sustained, 1300.0, {"reasons": []})[0] == burst
    assert bench.roofline_peak(burst, sustained, 1300.0, None)[0] == burst
