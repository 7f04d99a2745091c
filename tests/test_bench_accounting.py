"""The bench's work accounting on the CPU: the prefill FLOP count it divides
by matches a brute-force count of visible (query row, key) pairs, and the
launch count of a decode call matches its kernels (plan, decode, and the
partition merge only when a sequence can span two partitions)."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_prefill_flops_count_visible_pairs():
    rng = np.random.default_rng(5)
    for _ in range(20):
        nseq = int(rng.integers(1, 5))
        ctx = rng.integers(0, 300, size=nseq)
        n, hq, d = int(rng.integers(1, 40)), int(rng.choice([8, 32])), int(rng.choice([64, 128]))
        pairs = 0
        for c in ctx:
            for i in range(n):           # row i sits at position c + i ...
                for t in range(c + n):   # ... and sees keys 0 .. c + i
                    pairs += t <= c + i
        # q·Kᵀ and P·V: 2·d multiply-adds each, per pair and query head
        assert bench.prefill_flops(ctx, n, hq, d) == 4 * d * hq * pairs


def test_decode_launch_count():
    assert bench.decode_launches(32, 16, 512) == 2       # 512 tokens fit one partition: no merge
    assert bench.decode_launches(33, 16, 512) == 3       # a sequence can span two partitions
    assert bench.decode_launches(256, 16, 0) == 3        # automatic 512-token partitions
    assert bench.decode_launches(64, 8, 0) == 2
