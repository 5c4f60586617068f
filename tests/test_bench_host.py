"""Host-side decisions of bench.py (CPU only): which dense-FP4 roofline
denominator a GEMM chain is divided by, and which end-to-end form a line
reports."""
import bench

PEAKS = {"hbm_gbs": 6551.0, "bf16_tflops": 1644.1, "bf16_tflops_sustained": 1370.8}


def test_short_chain_takes_the_burst_figure():
    peak, regime = bench.tensor_peak(PEAKS, 19.5, [])
    assert regime == "burst"
    assert peak == PEAKS["bf16_tflops"] * bench.FP4_PER_BF16


def test_long_chain_or_power_cap_takes_the_sustained_figure():
    for chain_ms, reasons in ((2056.0, []), (1000.0, None), (19.5, ["sw_power_cap"])):
        peak, regime = bench.tensor_peak(PEAKS, chain_ms, reasons)
        assert regime == "sustained", (chain_ms, reasons)
        assert peak == PEAKS["bf16_tflops_sustained"] * bench.FP4_PER_BF16


def test_other_clock_reasons_do_not_change_the_regime():
    assert bench.tensor_peak(PEAKS, 999.0, ["hw_slowdown"])[1] == "burst"


def test_end_to_end_form_is_the_faster_one():
    assert bench.e2e_choice(15.5, 21.7) == (15.5, "pipelined")
    assert bench.e2e_choice(0.070, 0.038) == (0.038, "serial")
    assert bench.e2e_choice(1.0, 1.0) == (1.0, "pipelined")
