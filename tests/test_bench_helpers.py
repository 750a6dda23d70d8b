"""The bench's own bookkeeping, on CPU: which bf16 peak a timing is divided by, when the
recorded DRAM traffic of the forward GEMM is reported, and the clock sampler, run against
a fake NVML that offers read queries only (so any attempt to change a GPU setting would
fail the test)."""
import sys
import types

import pytest

import bench

PEAKS = {"hbm_gbs": 6538.3, "bf16_tflops": 1631.1, "bf16_tflops_sustained": 1375.3, "source": "measured",
         "sustained_sm_mhz": 1320.0}


def test_short_timed_region_takes_the_burst_peak():
    peak, why = bench.pick_tensor_peak(PEAKS, 0.035, {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert peak == 1631.1 and "burst" in why and "under 1 s" in why
    # short but power-capped: still timed as a burst
    peak, _ = bench.pick_tensor_peak(PEAKS, 0.5, {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]})
    assert peak == 1631.1


def test_long_region_at_max_clock_without_cap_is_a_burst():
    peak, why = bench.pick_tensor_peak(PEAKS, 4.0, {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": []})
    assert peak == 1631.1 and "no power cap" in why


def test_long_capped_region_takes_the_sustained_peak():
    for clk in ({"sm_mhz": 1740.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]},
                {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]},
                {"sm_mhz": 1500.0, "sm_max_mhz": 1965.0, "reasons": []}):
        peak, why = bench.pick_tensor_peak(PEAKS, 2.5, clk)
        assert peak == 1375.3 and "sustained" in why, clk


def test_without_a_sustained_figure_the_burst_is_used():
    peaks = dict(PEAKS, bf16_tflops_sustained=None)
    peak, why = bench.pick_tensor_peak(peaks, 5.0, {"sm_mhz": 1300.0, "sm_max_mhz": 1965.0,
                                                    "reasons": ["sw_power_cap"]})
    assert peak == 1631.1 and "no sustained figure" in why


def test_per_clock_rate_of_the_library_gemm():
    assert bench.cublas_tflops_per_ghz(PEAKS) == pytest.approx(1375.3 / 1.32)
    assert bench.cublas_tflops_per_ghz(dict(PEAKS, sustained_sm_mhz=None)) is None


def test_traffic_is_reported_only_for_the_sources_it_was_captured_on(monkeypatch):
    now = bench.sources_sha256_16(bench.FWD_MAIN_SOURCES)
    monkeypatch.setattr(bench, "FWD_MAIN_TRAFFIC", {"bytes": 123, "sources_sha256_16": now})
    assert bench.fwd_main_traffic() == 123
    monkeypatch.setattr(bench, "FWD_MAIN_TRAFFIC", {"bytes": 123, "sources_sha256_16": "0" * 16})
    assert bench.fwd_main_traffic() is None


class _FakeNvml(types.ModuleType):
    """Read-only NVML: clock, reasons, power. Nothing that sets anything exists here."""

    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonSwPowerCap = 0x4

    def __init__(self, clocks, reasons):
        super().__init__("pynvml")
        self._clocks, self._reasons, self.calls = list(clocks), list(reasons), []

    def __getattr__(self, name):
        raise AttributeError(f"the fake NVML has no {name}")

    def nvmlInit(self):
        self.calls.append("init")

    def nvmlDeviceGetHandleByUUID(self, uuid):
        self.calls.append("handle")
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls.append("clock")
        return self._clocks[min(len(self._clocks) - 1, self.calls.count("clock") - 1)]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self._reasons[min(len(self._reasons) - 1, self.calls.count("clock") - 1)]

    def nvmlDeviceGetPowerUsage(self, h):
        return 950_000


def test_clock_sampler_reports_median_and_reasons_with_read_queries_only(monkeypatch):
    fake = _FakeNvml([1740, 1750, 1730, 1740, 1745], [0x4, 0x0, 0x4, 0x4, 0x0])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(uuid="0123-4567"))
    s = bench.ClockSampler(0, period_s=0.001)
    import time
    t0 = time.time()
    while len(s.samples) < 5 and time.time() - t0 < 5:
        time.sleep(0.001)
    out = s.stop()
    assert s.err is None, s.err
    assert out["source"] == "nvml" and out["samples"] >= 5
    assert out["sm_max_mhz"] == 1965.0 and 1730 <= out["sm_mhz"] <= 1750 and out["sm_mhz_min"] == 1730
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 950.0
    assert set(fake.calls) <= {"init", "handle", "clock"}


def test_clock_sampler_flags_a_thermal_slowdown(monkeypatch):
    fake = _FakeNvml([1500], [0x40 | 0x4])
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.setattr(bench.torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(uuid="GPU-0123"))
    s = bench.ClockSampler(0, period_s=0.001)
    out = s.stop()
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
