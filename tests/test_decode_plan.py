"""Host-side rule that picks the e4m3 decode's automatic split count (CPU only).

bench.py restates the library's rule to report `config.num_splits`; these tests pin that
restatement against a direct list-scheduling estimate of the makespan, so that the rule
picks what it says it picks."""
import heapq
import math
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def makespan(units, nblk, n, slots, ovh=3):
    """Every (unit, split) CTA in launch order onto the first free slot of `slots`."""
    bps = -(-nblk // n)
    pieces = [min(bps, nblk - s * bps) + ovh for s in range(-(-nblk // bps))]
    free = [0] * slots
    heapq.heapify(free)
    end = 0
    for _ in range(units):
        for d in pieces:
            t = heapq.heappop(free) + d
            end = max(end, t)
            heapq.heappush(free, t)
    return end


def test_rule_matches_the_measured_best_counts_on_148_sms():
    # Llama-8B decode, Sk = 32768 (512 blocks), 8 KV heads, two CTAs per SM on 148 SMs
    picks = {B: bench.fp8_decode_splits(B * 8, 512, 296) for B in (1, 16, 64, 128, 256)}
    assert picks == {1: 37, 16: 9, 64: 4, 128: 2, 256: 1}


def test_rule_is_never_worse_than_whole_waves_of_one_or_two_ctas_per_sm():
    for units in (1, 8, 24, 128, 200, 512, 1000):
        for nblk in (4, 63, 512, 2048):
            n = bench.fp8_decode_splits(units, nblk, 296)
            assert 1 <= n <= max(1, min(64, nblk // 4))
            # the count the earlier rule took: splits that fill two CTAs per SM once
            old = max(1, min(64, 296 // units, max(1, nblk // 4)))
            assert makespan(units, nblk, n, 296) <= makespan(units, nblk, old, 296) * 1.02


def test_wave_estimate_agrees_with_the_list_schedule_for_equal_splits():
    # when n divides nblk all splits are equal and the estimate is exact
    for units, nblk, n in ((128, 512, 8), (512, 512, 4), (8, 512, 32), (1024, 512, 2)):
        bps = nblk // n
        est = math.ceil(units * n / 296) * (bps + 3)
        assert makespan(units, nblk, n, 296) == est
