"""Host logic of bench.py that needs no GPU: the clock record and the
algorithmic byte counts the roofline figures divide by."""
import bench


def test_parse_clocks_median_and_reasons():
    lines = [
        "index, clocks.current.sm, clocks.max.sm, power.draw, clocks_event_reasons.active, "
        "clocks_event_reasons.hw_slowdown, clocks_event_reasons.hw_thermal_slowdown, "
        "clocks_event_reasons.sw_thermal_slowdown, clocks_event_reasons.sw_power_cap",   # a header: skipped
        "0, 1965, 1965, 412.50, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1590, 1965, 998.10, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1605, 1965, 1001.30, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, [N/A], 1965, [N/A], [N/A], [N/A], [N/A], [N/A], [N/A]",                      # unreadable: skipped
        "0, 1650",                                                                        # short: skipped
    ]
    c = bench.parse_clocks(lines)
    assert c == {"sm_mhz": 1605.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_parse_clocks_reports_every_throttle_reason():
    line = "0, 1200, 1965, 700.0, 0x00000000000000E8, Active, Active, Active, Not Active"
    c = bench.parse_clocks([line])
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert bench.parse_clocks([]) is None


def test_workload_bytes_of_the_ffn_down_projection():
    m, k, n, r = 16384, 20480, 5120, 32
    by = bench.workload_bytes(m, k, n, r, m, with_w=False)
    # X read (2 B), codes (0.5 B) and scales (1/16 B) per element, D in fp32 per row
    assert by["quantize"] == 861_929_472 == m * k * 2 + m * k // 2 + m * k // 16 + m * r * 4
    assert by["calib"] == 671_088_640                 # X alone: the weight's absmax is stored
    assert by["score"] == 335_544_320                 # Yq and Yref, bf16
    assert bench.workload_bytes(m, k, n, r, m, with_w=True)["calib"] == 671_088_640 + n * k * 2
