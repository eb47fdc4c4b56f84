"""Host-side pieces of bench.py that need no GPU: the output check of the
CPU-baseline leg and the clock record of a timed region."""

import numpy as np

import bench


def test_output_check_bound_is_tolerance_plus_one_rounding():
    ref = np.array([[0.5, -1.0, 0.0]])
    # bf16 output (q format 1), 16-bit cache: 2e-3 + 2 * 2^-8 * |ref|
    ok, exc, err = bench.check_outputs(ref + np.array([[2e-3 + 2 * 2 ** -8 * 0.5 - 1e-9, 0.0, 0.0]]), ref, 1, 1)
    assert ok and exc < 0
    ok, exc, err = bench.check_outputs(ref + np.array([[0.0, 0.0, 2e-3 + 1e-6]]), ref, 1, 1)
    assert not ok and abs(err - (2e-3 + 1e-6)) < 1e-12
    # FP8 cache: 1e-2
    ok, _, _ = bench.check_outputs(ref + 9e-3, ref, 0, 2)
    assert ok


def test_clock_summary_keeps_only_samples_inside_the_region():
    clk = bench.ClockSampler.__new__(bench.ClockSampler)
    clk.ok, clk.max_mhz = True, 1965
    clk.samples = [(0.0, 500, 0x1), (1.0, 1965, 0x0), (1.5, 1900, 0x4), (2.0, 1965, 0x0), (3.0, 300, 0x1)]
    s = clk.summary(0.9, 2.1)
    assert s["samples"] == 3 and s["sm_mhz"] == 1965 and s["sm_min_mhz"] == 1900
    assert s["reasons"] == ["sw_power_cap"]
    assert clk.summary(5.0, 6.0)["samples"] == 0


def test_unique_and_logical_tokens_count_shared_blocks_once():
    tables = np.array([[7, 8, 9], [7, 8, 3]], np.int32)
    lens = np.array([40, 35], np.int32)  # block 16: blocks 7, 8 shared in full
    u, l = bench.unique_and_logical_tokens(tables, lens, 16)
    assert l == 75
    assert u == 16 + 16 + 8 + 3
