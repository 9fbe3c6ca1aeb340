"""Host logic of the memory-budget sweep (bench.py --budget-sweep): the batch
that fits a KV-cache budget for the 32-layer, n = 3328 InternVL-2.5-8B step."""

import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def test_cache_bytes_per_sequence():
    b1, b16, per1, per16 = bench.budget_batches(5)
    # 32 layers x 8 kv-heads x (K and V codes: 3328 tokens x 16 B, + alpha / step of K and V: 4 x 128 x 2 B)
    assert per1 == 32 * 8 * (2 * 3328 * 16 + 4 * 128 * 2) == 27_525_120
    # 32 layers x 8 kv-heads x K and V x 3328 x 128 x 2 B
    assert per16 == 32 * 8 * 2 * 3328 * 128 * 2 == 436_207_616
    assert per16 / per1 > 15.8  # 16x smaller codes, minus the statistics


def test_largest_batch_per_budget():
    got = [bench.budget_batches(gb)[:2] for gb in (5, 10, 20, 30)]
    assert got == [(181, 11), (363, 22), (726, 45), (1089, 68)]
    for gb, (b1, b16) in zip((5, 10, 20, 30), got):
        _, _, per1, per16 = bench.budget_batches(gb)
        assert b1 * per1 <= gb * 1e9 < (b1 + 1) * per1
        assert b16 * per16 <= gb * 1e9 < (b16 + 1) * per16
