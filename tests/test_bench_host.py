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
