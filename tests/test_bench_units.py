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
