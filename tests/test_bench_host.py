"""Host-side pieces of bench.py that need no GPU: the clock-record summary
that decides whether a timed run is kept, and the packed-byte count behind
every GB/s figure."""
import bench


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.lines = list(lines)
    return s


def test_clock_summary_median_max_and_reasons():
    # index, sm, max sm, power, active mask, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
    rows = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 950.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    ]
    got = _sampler(rows).summary()
    assert got == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_flags_every_rejecting_reason():
    rows = ["0, 1200, 1965, 500, 0x68, Active, Active, Active, Not Active"]
    got = _sampler(rows).summary()
    assert got["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_skips_short_and_unreadable_rows():
    rows = [
        "",
        "0, 1965",                                                    # cut short
        "0, [N/A], 1965, 1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1500, 1965, 1, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    got = _sampler(rows).summary()
    assert got["samples"] == 1 and got["sm_mhz"] == 1500.0 and got["reasons"] == []


def test_clock_summary_without_samples():
    assert _sampler([]).summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_layer_packed_bytes_per_token():
    # one P=4 expert: 3 matrices of 2048 x 1408 weights at 4.5 bytes per
    # 8-weight block (2 seed + 2 coefficient + 0.5 code bytes) = 4,866,048 B,
    # plus an int32 exponent bias per row (1408 + 1408 + 2048 rows); a token
    # reads 8 experts per layer
    expert = 3 * 2048 * 1408 // 8 * 9 // 2 + 4 * (1408 + 1408 + 2048)
    assert 3 * 2048 * 1408 // 8 * 9 // 2 == 4_866_048
    assert bench.layer_packed_bytes_per_token() == 8 * expert == 39_084_032
