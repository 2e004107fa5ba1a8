"""bench.py's work accounting, pinned by counting (no GPU)."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_causal_attention_flops_counts_visible_pairs():
    """2 products x 2 FLOPs per multiply-add x D, over every (query i, key j <= i) pair of
    every (sequence, query head): counted pair by pair on small prompts."""
    for B, Hq, D, S in [(1, 1, 1, 1), (2, 3, 64, 7), (1, 4, 128, 130)]:
        pairs = sum(1 for i in range(S) for j in range(S) if j <= i)
        assert bench.causal_attention_flops(B, Hq, D, S) == 2 * 2 * B * Hq * D * pairs
    # one Llama-3-8B layer, 8K prompt, batch 4: 2.199 TFLOP
    assert abs(bench.causal_attention_flops(4, 32, 128, 8192) / 1e12 - 2.1993) < 1e-3
