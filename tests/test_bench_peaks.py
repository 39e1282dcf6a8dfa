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
