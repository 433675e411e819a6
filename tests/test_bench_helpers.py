"""Host logic of bench.py that needs no GPU: the traffic figure is reported only
while the kernel sources are the ones the committed ncu summary was taken on, the
roofline peak comes from the measured peaks file, and the clock record is parsed
into the median SM clock and the throttle reasons seen."""
import bench


def test_profiled_traffic_tracks_the_kernel_sources(monkeypatch):
    import re
    text = open(bench.PROFILE_FILE).read()
    profiled = re.search(r"kernel_source_sha256_16:\s*([0-9a-f]+)", text).group(1)
    # on the sources the summary was captured on, its DRAM bytes per launch are reported
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: profiled)
    got = bench.profiled_traffic()
    assert isinstance(got, int) and got > 2_000_000_000
    # on any other sources, none
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic() is None


def test_peak_is_the_measured_copy_bandwidth():
    peak, kind = bench.hbm_peak()
    assert kind == "measured" and 5000.0 < peak < 8000.0


def test_clock_summary_takes_median_and_reasons():
    c = bench.ClockSampler(0)
    c.lines = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = c.summary()
    assert s["sm_mhz"] == 1900.0 and s["sm_max_mhz"] == 1965.0
    assert s["reasons"] == ["sw_power_cap"] and s["samples"] == 3
    assert bench.ClockSampler(0).summary()["sm_mhz"] is None
