"""The bench's host-side measurement logic on the CPU: the nvidia-smi clock
record (filtered to the timed GPU, throttle reasons, the loaded SM clock)
and the L2-rotation set count."""
import bench

# uuid, index, clocks.sm, clocks.max.sm, power.draw, hw_slowdown,
# hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
ROWS = """GPU-aaaa, 0, 1965, 1965, 610.5, Not Active, Not Active, Not Active, Active
GPU-bbbb, 1, 1200, 1965, 300.0, Active, Not Active, Not Active, Not Active
GPU-aaaa, 0, 1500, 1965, 990.0, Not Active, Not Active, Not Active, Active
GPU-aaaa, 0, 345, 1965, 90.0, Not Active, Not Active, Not Active, Not Active
GPU-aaaa, 0, 1965, 1965, 400.0, Not Active, Not Active, Not Active, Not Active
"""


def test_clocks_filtered_to_the_timed_gpu():
    c = bench.ClockSampler("GPU-AAAA", "7").parse(ROWS)
    # GPU 1's hw_slowdown is not ours; idle samples (345 MHz) are left out of
    # the loaded median and minimum
    assert c["reasons"] == ["sw_power_cap"]
    assert c["samples"] == 4
    assert c["sm_mhz"] == 1965.0 and c["sm_mhz_min"] == 1500.0
    assert c["sm_max_mhz"] == 1965.0 and c["power_w_max"] == 990.0


def test_clocks_by_index_without_uuid():
    c = bench.ClockSampler("", "1").parse(ROWS)
    assert c["reasons"] == ["hw_slowdown"] and c["samples"] == 1 and c["sm_mhz_min"] == 1200.0


def test_clocks_unsampled():
    c = bench.ClockSampler("GPU-cccc", "5").parse("")
    assert c["reasons"] == ["unsampled"] and c["samples"] == 0


def test_rotation_sets_cover_three_l2():
    for nbytes in (1, 10 << 20, bench.L2_BYTES, 5 * bench.L2_BYTES):
        n = bench._nsets(nbytes)
        assert n >= 2 and n * nbytes >= 3 * bench.L2_BYTES
        assert (n - 1) * nbytes < 3 * bench.L2_BYTES or n == 2


def _fake_line():
    bw = {"ms": 0.0123456, "GB/s": 6000.0, "hbm_frac": 0.93}
    sweep = {str(m): {"ms": 0.01 * (1 + m / 512), "roofline_frac": 0.8} for m in (1, 64, 512, 4608, 16384)}
    wo = {k: {"ms": 0.1, "frac_bf16_burst": 0.9} for k in ("bf16_gemm", "float8", "gguf")}
    extras = {"quantize_rows_4608x12288": bw, "q8_0_quantize_2^28": bw, "q8_0_dequantize_2^28": bw,
              "q8_0_to_axis_int8_12288x3072": bw, "q8_0_to_axis_e4m3_12288x3072": bw,
              "dequantize_e4m3_bf16_12288x3072": bw, "q8_0_dequantize_bf16_12288x3072": bw,
              "quantize_weight_tensor_12288x3072": {"ms": 0.03, "GB/s": 3000.0},
              "int_w8a8_fwd_tiny_256x512x512": {"ms": 0.005},
              "float_w8a8_fwd_4096x3072x3072": {"ms": 0.04, "TOPS": 1900.0, "gemm_ms": 0.03,
                                                "gemm_frac_fp8_burst": 0.75},
              "svdquant_r32_fwd_4608x3072x3072": {"ms": 0.04, "frac_int8_burst": 0.6},
              "svdquant_e4m3_r32_fwd_4608x3072x3072": {"ms": 0.045, "frac_fp8_burst": 0.55},
              "gguf_a8_int_fwd_sweep_N12288_K3072": sweep, "gguf_a8_float_fwd_sweep_N12288_K3072": sweep,
              "weight_only_fwd_4608x12288x3072": wo, "weight_only_dgrad_4608x12288x3072": wo,
              "dit_mlp_fwd_gelu_4608x3072x12288": {"unfused": {"ms": 0.28}, "fused_absmax": {"ms": 0.281}}}
    return {"value": 2757.123, "ms_per_step": 0.50474, "roofline": {"frac": 0.97294},
            "e2e": {"value": 1077.0}, "extras": extras}


def test_summary_rows_are_short_and_cover_every_row():
    """The bench line ends with the per-row summary; it stays short enough to
    survive a reader that keeps only the last ~3000 characters of output."""
    import json
    rows = bench.summary_rows(_fake_line())
    text = json.dumps({"rows": rows})
    assert len(text) < 2500, len(text)
    for key in ("headline_dit_mlp_fwd_dgrad", "a1_quantize_rows_4608x12288", "a3_q8_0_quantize_2^28",
                "a3_q8_0_dequantize_2^28", "a4_q8_0_to_axis_int8_12288x3072", "cfg1_int_tiny_256x512x512",
                "cfg2_float_w8a8_4096x3072x3072", "cfg4_svdquant_int8_r32", "cfg5_gguf_a8_int",
                "f2_gguf_a8_float", "f3_weight_only_frac_bf16", "f4_svdquant_e4m3_r32", "f1_mlp_fwd_gelu_us"):
        assert key in rows
    assert rows["headline_dit_mlp_fwd_dgrad"]["TOPS"] == 2760.0      # 3 significant digits
    assert set(rows["cfg5_gguf_a8_int"]) == {"1", "64", "512", "4608", "16384"}
