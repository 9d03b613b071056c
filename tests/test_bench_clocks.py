"""bench.py's clock summary (host logic, no GPU): samples inside the timed window,
widening of a window too short to hold any, and the throttle reasons it reports."""

import bench


def _sampler(samples, window, max_mhz=1965):
    s = bench.ClockSampler.__new__(bench.ClockSampler)
    s.samples, s.window, s.max_mhz, s.error = samples, window, max_mhz, None
    return s


def test_median_inside_the_window():
    smp = [(t, 1965 if t >= 10 else 1200, 0) for t in range(0, 20)]
    out = _sampler(smp, (10.0, 19.0)).summary()
    assert out["sm_mhz"] == 1965 and out["samples"] == 10 and "window_padded_ms" not in out


def test_short_window_is_widened_to_neighbouring_samples():
    # samples every 20 ms, a 5 ms window between two of them
    smp = [(1.000 + 0.02 * i, 1965, 0x4 if i == 3 else 0) for i in range(10)]
    out = _sampler(smp, (1.062, 1.067)).summary()
    assert out["samples"] >= 3 and out["sm_mhz"] == 1965 and out["window_padded_ms"] > 0
    assert out["reasons"] == ["sw_power_cap"]


def test_no_samples_at_all():
    out = _sampler([], (1.0, 1.1)).summary()
    assert out["sm_mhz"] is None and out["samples"] == 0
