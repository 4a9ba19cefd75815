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


def test_every_page_configuration_is_measured():
    """The headline (prefill) plus the workloads object cover every configuration of the pages:
    the 64x2112x7168 C = 0 decode shape, decode M = 64 and 128 cold and warm, contiguous, masked."""
    keys = {k for k, _, _ in bench.SUB_WORKLOADS}
    assert {"config1", "decode64_cold", "decode64_warm", "decode128_cold", "decode128_warm",
            "contiguous", "masked"} <= keys
    # and the rows beyond the page configurations: the other layouts and the K-grouped GEMM
    assert {"layouts", "k_grouped"} <= keys
    c1 = bench.WORKLOADS["config1"]
    assert c1["M"] == 64 and c1["shapes"] == [(2112, 7168)] and not c1["with_c"]
    for name in ("decode64", "decode128"):
        assert bench.WORKLOADS[name]["shapes"] == bench.PREFILL_SHAPES
    assert bench.WORKLOADS["contiguous"]["G"] == 8 and bench.WORKLOADS["masked"]["G"] == 16


def test_algorithmic_bytes_of_the_decode_headline_shape():
    """64x2112x7168 with C = 0: A and B e4m3, their fp32 scales, D bf16 (15.9 MB)."""
    p = {"kind": "dense", "rows": 64, "N": 2112, "K": 7168, "G": 1, "with_c": False}
    kb, nb = 56, 17
    assert bench.algorithmic_bytes(p) == 64 * 7168 + 4 * 64 * kb + 2112 * 7168 + 4 * nb * kb + 2 * 64 * 2112


def test_stored_traffic_is_dropped_when_the_kernels_change(tmp_path, monkeypatch):
    import json
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "source_digest", lambda: "f" * 40)     # the current kernels' digest
    (prof / "traffic.json").write_text(json.dumps({
        "prefill": {"bytes_per_launch": 123.0, "source_sha1": "f" * 40},
        "decode64": {"bytes_per_launch": 7.0, "source_sha1": "0" * 40}}))
    assert bench.stored_traffic("prefill") == 123.0
    assert bench.stored_traffic("decode64") is None
    assert bench.stored_traffic("masked") is None


def test_k_grouped_problem_sizes_and_bytes():
    """The K-grouped workload: G = 8 groups of U{2048..6144} tokens padded to 128, gradient
    shapes (M,N) from the expert weights; bytes = both e4m3 operands, their per-channel scales
    and the fp32 D."""
    probs = bench.make_problems(dict(bench.WORKLOADS["k_grouped"], shapes=[(256, 128)]))
    (p,) = probs
    assert len(p["ks"]) == 8 and all(k % 128 == 0 and 2048 <= k <= 6144 + 127 for k in p["ks"])
    T = sum(p["ks"])
    assert p["K"] == T and p["x"].shape == (T, 256) and p["w"].shape == (T, 128)
    assert p["flops"] == 2.0 * 256 * 128 * T
    assert bench.algorithmic_bytes(p) == T * 256 + T * 128 + 4 * (T // 128) * (256 + 128) + 4 * 8 * 256 * 128
