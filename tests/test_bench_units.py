"""The algorithmic units behind every rate bench.py reports, checked against
numbers that do not come from bench.py: the golden window counts (derived from
b = 128, s = 1, l = 7) and the oracle's own per-query key counts."""
import json
import os

import pytest

import bench

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "window_counts.json")


def test_prefill_flops_use_the_golden_pair_counts():
    pairs = json.load(open(GOLDEN))["pairs_per_sequence"]
    for L, n in pairs.items():
        # 2 (d_qk + d_v) FLOP per visible (query, key) pair per head, 64 heads, 576 + 512
        assert bench.prefill_flops(int(L)) == 2 * (576 + 512) * 64 * n


def test_decode_bytes_read_each_selected_row_once(oracle_mod):
    lens = [1, 127, 128, 129, 1024, 1025, 5000, 65536, 131072]
    rows = sum(oracle_mod.visible_count(L - 1, 128, 1, 7) for L in lens)
    per_seq = 64 * (576 * 2 + 512 * 2 + 4)  # q, out (bf16) and lse (fp32) of 64 heads
    assert bench.decode_bytes(lens) == rows * 1152 + len(lens) * per_seq


def test_dense_decode_bytes_read_the_whole_context():
    lens = [1, 700, 131072]
    assert bench.decode_bytes(lens, n_local=-1) == sum(lens) * 1152 + len(lens) * 64 * (576 * 2 + 512 * 2 + 4)


@pytest.mark.parametrize("L", [1024, 2048, 32768])
def test_window_rows_never_exceed_the_window(oracle_mod, L):
    assert bench.decode_bytes([L]) <= 1024 * 1152 + 64 * (576 * 2 + 512 * 2 + 4)


@pytest.mark.parametrize("L", [1, 15, 16, 17, 1024, 1040, 1041, 5000, 1 << 20])
def test_hi_window_rows_are_the_token_windows_keys(oracle_mod, L):
    """The HI line's window part: the keys of the last token under page 4's
    16 sink tokens + 1,024-token window (b = 1), as the oracle counts them."""
    assert bench.token_window_rows(L) == oracle_mod.visible_count(L - 1, 1, 16, 1024)


def test_job_value_is_all_ranks_work_over_the_slowest_time():
    # 4 ranks x 5 steps x 2 units of work, the slowest rank taking 250 ms: 160 units/s
    assert bench.job_value(4, 5, 2.0, 250.0) == pytest.approx(160.0)
    assert bench.job_value(1, 5, 2.0, 250.0) == pytest.approx(40.0)


def test_rooflines_divide_the_algorithmic_rate_by_the_measured_peaks():
    peaks = {"bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6500.0}
    r = bench.tensor_roofline(4e12, 4.0, peaks, "measured", "no_such_kernel")
    assert r["achieved"] == pytest.approx(1000.0) and r["frac"] == pytest.approx(1000.0 / 1600.0)
    assert r["peak"] == 1600.0 and r["traffic"] is None  # no ncu record for this kernel
    s = bench.tensor_roofline(4e12, 4.0, peaks, "measured", "no_such_kernel", sustained=True)
    assert s["peak"] == 1400.0 and s["frac"] == pytest.approx(1000.0 / 1400.0)
    assert s["frac_of_burst"] == pytest.approx(1000.0 / 1600.0)
    h = bench.hbm_roofline(6.5e9, 2.0, peaks, "measured", "no_such_kernel")
    assert h["achieved"] == pytest.approx(3250.0) and h["frac"] == pytest.approx(0.5) and h["unit"] == "GB/s"
