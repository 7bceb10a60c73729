"""Host-side pieces of bench.py that decide whether a number is kept, without a GPU: the clock
record (median SM clock and the throttle reasons seen inside the timed region) and the ncu
traffic lookup, which must only report counters taken on the current kernel source."""
import bench


def _row(sm, reasons_active=()):
    names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
    flags = ["Active" if n in reasons_active else "Not Active" for n in names]
    return ", ".join(["2026/01/01 00:00:00.000", str(sm), "1965", "700.0", "0x0"] + flags)


def test_clock_record_keeps_only_the_timed_region():
    s = bench.ClockSampler("0")
    s.lines = [(0.0, _row(1965)),                                  # before: idle, full clock
               (10.0, _row(1500, ["sw_power_cap"])),
               (10.5, _row(1520, ["sw_power_cap"])),
               (11.0, _row(1540)),
               (20.0, _row(800, ["hw_slowdown"]))]                  # after the timed region
    s.t0, s.t1 = 9.9, 11.05
    rec = s.stop()
    assert rec["samples_in_timed_region"] == 3
    assert rec["sm_mhz"] == 1520 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]                      # hw_slowdown was outside


def test_clock_record_reports_rejecting_reasons():
    s = bench.ClockSampler("0")
    s.lines = [(1.0, _row(1200, ["hw_thermal_slowdown"])), (1.1, "garbage"), (1.2, _row(1300))]
    s.t0, s.t1 = 0.9, 1.3
    rec = s.stop()
    assert rec["reasons"] == ["hw_thermal_slowdown"] and rec["samples_in_timed_region"] == 2


def test_traffic_only_for_the_current_kernel_source():
    for k in bench.KERNEL_FILES:
        h = bench.kernel_source_hash(k)
        assert len(h) == 16 and h == bench.kernel_source_hash(k)
        t = bench.measured_traffic(k)
        assert t is None or t > 0
    assert bench.kernel_source_hash("window_attn_kernel") != bench.kernel_source_hash("append_fill")
