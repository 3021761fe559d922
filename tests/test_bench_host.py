"""Host-side arithmetic of bench.py (no GPU)."""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


def test_prefill_flops_counts_causal_pairs():
    # brute force: every (new token, key <= its position) pair
    rng = np.random.default_rng(0)
    lengths = rng.integers(1, 300, size=7)
    q_lens = [int(rng.integers(0, L + 1)) for L in lengths]
    pairs = sum(1 for L, n in zip(lengths, q_lens)
                for p in range(L - n, L) for _ in range(p + 1))
    assert bench.prefill_flops(lengths, q_lens, 6, 64) == 4 * 64 * 6 * pairs


def test_prefill_flops_closed_forms():
    # whole prompt: L(L+1)/2 pairs; one new token: L pairs (decode)
    assert bench.prefill_flops([4096], [4096], 1, 1) == 4 * 4096 * 4097 // 2
    assert bench.prefill_flops([4096], [1], 1, 1) == 4 * 4096
    assert bench.prefill_flops([10], [0], 3, 8) == 0


def test_kv_bytes():
    from paged_kv_cache_383_b200 import workloads as wl
    w = wl.WORKLOADS["llama3_70b_gqa8"]
    assert bench.kv_bytes([1, 2], w) == 3 * 8 * 128 * 2 * 2
