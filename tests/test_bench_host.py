"""Host-side logic of bench.py that needs no GPU: the tensor peak chosen from the sampled clocks,
and the kernel each problem takes under the library's documented dispatch rule."""
import bench

PEAKS = {"hbm_gbs": 6541.8, "bf16_tflops": 1624.0, "bf16_tflops_sustained": 1366.7}


def test_full_clock_takes_the_burst_peak():
    peak, kind = bench.fp8_tensor_peak(PEAKS, {"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []})
    assert peak == 2 * 1624.0 and kind.startswith("bf16_tflops (burst")


def test_power_cap_takes_the_sustained_peak():
    peak, kind = bench.fp8_tensor_peak(PEAKS, {"sm_mhz": 1717, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]})
    assert peak == 2 * 1366.7 and kind.startswith("bf16_tflops_sustained")
    # a power-cap reason alone is enough, even at a clock near the maximum
    assert bench.fp8_tensor_peak(PEAKS, {"sm_mhz": 1950, "sm_max_mhz": 1965,
                                         "reasons": ["sw_power_cap"]})[0] == 2 * 1366.7


def test_low_clock_without_a_reason_takes_the_sustained_peak():
    assert bench.fp8_tensor_peak(PEAKS, {"sm_mhz": 1500, "sm_max_mhz": 1965, "reasons": []})[0] == 2 * 1366.7


def test_no_clock_samples_take_the_burst_peak():
    assert bench.fp8_tensor_peak(PEAKS, {"sm_mhz": None, "sm_max_mhz": None, "reasons": []})[0] == 2 * 1624.0


def test_missing_sustained_figure_falls_back_to_burst():
    peaks = {"hbm_gbs": 1.0, "bf16_tflops": 100.0}
    assert bench.fp8_tensor_peak(peaks, {"sm_mhz": 1000, "sm_max_mhz": 1965, "reasons": []})[0] == 200.0


def test_kernel_names_follow_the_dispatch_rule():
    dense = lambda M, N, K: {"kind": "dense", "rows": M, "N": N, "K": K}
    # at most 128 rows: cluster split-K for <= 64 weight tiles and K <= 8192, else stream-K
    assert bench.gemm_kernel_name(dense(64, 2112, 7168)) == "gemm_splitk_kernel"
    assert bench.gemm_kernel_name(dense(128, 8192, 8192)) == "gemm_splitk_kernel"
    assert bench.gemm_kernel_name(dense(128, 8193, 8192)) == "gemm_swap_kernel"      # 65 tiles
    assert bench.gemm_kernel_name(dense(64, 7168, 16384)) == "gemm_swap_kernel"      # Kb = 128
    assert bench.gemm_kernel_name(dense(64, 24576, 1536)) == "gemm_swap_kernel"      # 192 tiles
    # more rows, and the grouped layouts: the tile kernel
    assert bench.gemm_kernel_name(dense(129, 2112, 7168)) == "gemm_kernel"
    assert bench.gemm_kernel_name({"kind": "masked", "rows": 256, "N": 4096, "K": 7168}) == "gemm_kernel"
    assert bench.gemm_kernel_name({"kind": "contiguous", "rows": 32768, "N": 4096, "K": 7168}) == "gemm_kernel"
