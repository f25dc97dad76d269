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


def test_cpu_baseline_reports_every_config_on_all_cores_and_one():
    # the oracle baseline: the seed GEMVs (512 x 1024 and the expert-sized
    # sweep, P=4 and P=3), one decode layer and the 45-layer stack, each with
    # all threads and with one, plus the host's core count and CPU model
    got = bench.cpu_baseline(budget_s=0.5)
    assert got["kind"] == "oracle" and got["unit"] == "tokens/s" and got["value"] > 0
    assert got["nproc"] >= 1 and got["cpu_model"] and got["cores"] >= 1
    assert got["all_cores"]["threads"] == got["cores"] and got["one_core"]["threads"] == 1
    for run in (got["all_cores"], got["one_core"]):
        shapes = {(g["P"], g["N"], g["K"]) for g in run["gemv"]}
        assert (4, 512, 1024) in shapes
        assert all((Pv, N, K) in shapes for Pv in (3, 4) for N, K in bench.GEMV_SHAPES)
        assert all(g["weights_per_s"] > 0 and g["packed_GB_s"] > 0 for g in run["gemv"])
        assert run["one_layer"]["tokens_per_s"] > 0 and run["stack"]["tokens_per_s"] > 0
    assert got["value"] == got["all_cores"]["stack"]["tokens_per_s"]


def test_clock_sampler_rows_from_nvml_reason_bits():
    # the NVML poller writes rows in nvidia-smi's field order, one Active flag
    # per reason bit (hw_slowdown 0x8, hw_thermal 0x40, sw_thermal 0x20,
    # sw_power_cap 0x4), which summary() reads back
    s = bench.ClockSampler(0)
    for sm, mask in ((1965, 0x0), (1850, 0x4), (1900, 0x4)):
        flags = ", ".join("Active" if mask & b else "Not Active" for b in bench.ClockSampler.BITS)
        s.lines.append(f"0, {sm}, 1965, 900.0, {mask:#x}, {flags}")
    assert s.summary() == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_sampler_keeps_only_the_timed_window():
    # samples stamped by the poller process before and after the timed region
    # are dropped; those inside it are summarised
    s = bench.ClockSampler(0)
    row = "0, {}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    s.stamped = [(0.5, row.format(1200)), (1.0, row.format(1965)), (1.2, row.format(1950)), (2.5, row.format(700))]
    s.t0, s.t1 = 0.9, 2.0
    s.keep_window()
    assert s.summary() == {"sm_mhz": 1957.5, "sm_max_mhz": 1965.0, "reasons": [], "samples": 2}


def test_layer_record_holds_only_for_the_sources_it_names(tmp_path):
    import bench
    d = bench.kernel_sources_sha256()
    assert len(d) == 64 and d == bench.kernel_sources_sha256()
    good = tmp_path / "rec.txt"
    good.write_text(f"dram_bytes_per_layer_call: 123\nwarp_instructions_per_layer_call: 45\n"
                    f"kernel_sources_sha256: {d}\n# a comment: 7\n")
    r = bench.layer_record(str(good))
    assert r == {"matches": True, "dram_bytes_per_layer_call": 123, "warp_instructions_per_layer_call": 45}
    stale = tmp_path / "stale.txt"
    stale.write_text("dram_bytes_per_layer_call: 123\nkernel_sources_sha256: unrecorded\n")
    r = bench.layer_record(str(stale))
    assert r["matches"] is False and r["warp_instructions_per_layer_call"] is None
    assert bench.layer_record(str(tmp_path / "missing.txt"))["matches"] is False


def test_gemv_shapes_option_parses_and_rejects():
    import argparse

    import pytest

    assert bench._gemv_shapes("8192x8192") == [(8192, 8192)]
    assert bench._gemv_shapes("2048X4096,1408x2048") == [(2048, 4096), (1408, 2048)]
    for bad in ("0x64", "16x12", "16x0", "16"):
        with pytest.raises((argparse.ArgumentTypeError, ValueError)):
            bench._gemv_shapes(bad)
