"""The bench's clock sampler against a fake NVML (no GPU, nothing on the device
is read or changed): samples are taken only between begin() and end(), samples
the driver flags as idle stay out of the median under load, and the reason bits
map to the names the bench reports."""
import time
import types

import bench


def _fake_nvml(clock_seq, reason_seq):
    calls = {"clock": 0, "reasons": 0}

    def clock(h, kind):
        assert h == "gpu" and kind == nv.NVML_CLOCK_SM
        v = clock_seq[min(calls["clock"], len(clock_seq) - 1)]
        calls["clock"] += 1
        return v

    def reasons(h):
        v = reason_seq[min(calls["reasons"], len(reason_seq) - 1)]
        calls["reasons"] += 1
        return v

    nv = types.SimpleNamespace(
        NVML_CLOCK_SM=1,
        nvmlClocksEventReasonGpuIdle=0x1,
        nvmlClocksEventReasonSwPowerCap=0x4,
        nvmlClocksEventReasonHwSlowdown=0x8,
        nvmlClocksEventReasonSwThermalSlowdown=0x20,
        nvmlClocksEventReasonHwThermalSlowdown=0x40,
        nvmlClocksEventReasonHwPowerBrakeSlowdown=0x80,
        nvmlDeviceGetClockInfo=clock,
        nvmlDeviceGetMaxClockInfo=lambda h, kind: 1965,
        nvmlDeviceGetCurrentClocksEventReasons=reasons,
    )
    return nv, calls


def _run(sampler, seconds):
    with sampler as s:
        time.sleep(0.01)                  # before the region: no samples
        n_before = len(s.rows)
        s.begin()
        time.sleep(seconds)
        s.end()
        n_region = len(s.rows)
        time.sleep(0.01)                  # after the region: no more samples
        n_after = len(s.rows)
    return n_before, n_region, n_after


def test_samples_only_inside_the_region_and_reasons_by_name():
    nv, _ = _fake_nvml([1965], [0x4])
    s = bench.ClockSampler(0)
    s._nvml = lambda: (nv, "gpu")
    n_before, n_region, n_after = _run(s, 0.03)
    assert n_before == 0
    assert n_region >= 3
    assert n_after <= n_region + 1          # at most the sample in flight at end()
    out = s.summary()
    assert out["sm_mhz"] == 1965 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == len(s.rows)
    assert "NVML" in out["source"]


def test_idle_samples_are_left_out_of_the_median():
    # the first two samples are idle at a low clock, the rest under load
    nv, _ = _fake_nvml([345, 345] + [1965] * 1000, [0x1, 0x1] + [0x0] * 1000)
    s = bench.ClockSampler(0)
    s._nvml = lambda: (nv, "gpu")
    _run(s, 0.03)
    out = s.summary()
    assert out["sm_mhz"] == 1965
    assert out["samples"] == len(s.rows) - 2
    assert out["reasons"] == []


def test_throttle_reasons_are_all_reported():
    nv, _ = _fake_nvml([1500], [0x8 | 0x20 | 0x40 | 0x80])
    s = bench.ClockSampler(0)
    s._nvml = lambda: (nv, "gpu")
    _run(s, 0.02)
    assert s.summary()["reasons"] == ["hw_power_brake_slowdown", "hw_slowdown",
                                      "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_without_nvml_or_nvidia_smi_the_summary_says_so(monkeypatch):
    s = bench.ClockSampler(0)
    s._nvml = lambda: (None, None)
    monkeypatch.setenv("PATH", "/nonexistent")
    with s:
        s.begin()
        s.end()
    assert s.summary()["sm_mhz"] is None
