"""bench.py's choice of the tensor roofline peak from the clocks sampled in the timed steps (CPU)."""
import bench

PEAKS = dict(hbm_gbs=6545.3, bf16_tflops=1639.1, bf16_tflops_sustained=1386.2, source="measured")


def test_burst_peak_without_power_cap():
    assert bench.choose_tc_peak(PEAKS, {"sm_mhz": 1965, "reasons": []}) == (1639.1, "bf16_tflops")


def test_sustained_peak_when_power_cap_was_sampled():
    clk = {"sm_mhz": 1200, "reasons": ["sw_power_cap"]}
    assert bench.choose_tc_peak(PEAKS, clk) == (1386.2, "bf16_tflops_sustained")


def test_unsampled_clocks_take_the_burst_peak():
    assert bench.choose_tc_peak(PEAKS, {"sm_mhz": None, "reasons": ["unsampled"]})[1] == "bf16_tflops"


def test_fraction_recomputes_from_flop_time_and_peak():
    # 6*T*k*H*I of the fine-grained workload over a 10 ms kernel against the burst peak
    flop = 6.0 * 16384 * 8 * 7168 * 2048
    achieved = flop / 10e-3 / 1e12
    peak, _ = bench.choose_tc_peak(PEAKS, {"reasons": []})
    assert abs(achieved / peak - 11.544e12 / 10e-3 / 1e12 / 1639.1) < 1e-3


def test_traffic_rows_count_only_for_the_current_kernel_source(tmp_path):
    table = tmp_path / "traffic.txt"
    table.write_text("# workload  hash  bytes  capture\n"
                     "mixtral  aaaa  100  full\n"
                     "mixtral  bbbb  200  full\n"
                     "mixtral+shared1  bbbb  300  full\n"
                     "skewed  aaaa  400  full\n")
    assert bench.measured_traffic("mixtral", str(table), "bbbb") == 200
    assert bench.measured_traffic("mixtral+shared1", str(table), "bbbb") == 300
    assert bench.measured_traffic("skewed", str(table), "bbbb") is None      # captured on another source
    assert bench.measured_traffic("decode", str(table), "bbbb") is None      # never captured
    assert bench.measured_traffic("mixtral", str(tmp_path / "none.txt"), "bbbb") is None


def test_committed_traffic_table_parses():
    import os
    rows = [l.split() for l in open(os.path.join(bench.ROOT, "profiles", "traffic.txt"))
            if l.strip() and not l.startswith("#")]
    assert rows and all(len(r) >= 3 and len(r[1]) == 16 and int(r[2]) > 0 for r in rows)
