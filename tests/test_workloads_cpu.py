"""The input recipes' helpers that the bench relies on."""

import numpy as np

from workloads import WORKLOADS, _TAG_K, _per_block, _rng, needle_block_list, needle_blocks


def test_needle_block_list_replays_the_key_generator():
    w = WORKLOADS["batched_needles_32k"].scaled(batch=3)
    n_blocks = -(-w.seq_len // w.block)
    for b, h in [(0, 0), (1, 3), (2, 7)]:
        _, spread = _per_block(_rng(w, _TAG_K, b, h), n_blocks, w.block, w.head_dim, w.keys)
        want = needle_blocks(w, b, h, spread)
        got = needle_block_list(w, b, h)
        assert np.array_equal(got, want)
        assert len(got) == w.needles
        # away from the sink and the local window, distinct
        assert got.min() >= w.sink_blocks
        assert got.max() < (w.seq_len - w.local_tokens) // w.block
        assert len(set(got.tolist())) == w.needles


def test_no_needles_elsewhere():
    assert len(needle_block_list(WORKLOADS["single_32k"], 0, 0)) == 0
