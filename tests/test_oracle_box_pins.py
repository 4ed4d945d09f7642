"""Pins of the oracle's min/max box selector against what fixes it from outside
the oracle: the box really bounds the keys and is attained by them; its score
is the brute-force maximum of q.k over the box's corners (a linear function
peaks at a corner); it bounds the exact log attention mass of the block from
above (the oracle-sparse mass, itself pinned against dense attention) and
equals it for a block of identical keys; and with the box selector as score
the selection obeys the same top-k / sink / local rules."""

import itertools
import math

import numpy as np
import pytest

import oracle.cobs_oracle as O


def test_box_bounds_and_touches_every_key_dimension():
    rng = np.random.default_rng(0)
    keys = rng.normal(size=(64, 32))
    lo, hi = O.block_box(keys)
    assert np.all(keys >= lo) and np.all(keys <= hi)
    for t in range(32):                       # each end is some key's value
        assert lo[t] in keys[:, t] and hi[t] in keys[:, t]


def test_score_is_the_maximum_over_the_corners():
    rng = np.random.default_rng(1)
    d = 8
    for _ in range(20):
        keys = rng.normal(size=(64, d)) * rng.uniform(0.1, 3.0)
        lo, hi = O.block_box(keys)
        q = rng.normal(size=d)
        best = max(float(np.dot(q, np.where(np.array(c), hi, lo)))
                   for c in itertools.product([0, 1], repeat=d))
        s = O.box_head_scores(q, lo[None], hi[None], np.array([64]))[0]
        assert abs(s - (math.log(64) + best / math.sqrt(d))) <= 1e-12 * max(1.0, abs(s))


def test_score_bounds_the_exact_log_mass_from_above():
    rng = np.random.default_rng(2)
    d, B = 64, 64
    keys = O.round_to_bf16(rng.normal(0.0, 0.5, size=(8 * B, d)))
    lo, hi = O.build_block_boxes(keys, B, 0, 8)
    for _ in range(10):
        q = rng.normal(size=d)
        exact = O.osa_head_masses(q[None], keys, 8 * B, B, 1.0 / math.sqrt(d))[0]
        box = O.box_head_scores(q, lo, hi, np.full(8, B))
        assert np.all(box >= exact - 1e-12)


def test_identical_keys_make_the_bound_exact():
    rng = np.random.default_rng(3)
    d, B = 16, 64
    k = rng.normal(size=d)
    keys = np.tile(k, (B, 1))
    lo, hi = O.block_box(keys)
    q = rng.normal(size=d)
    s = O.box_head_scores(q, lo[None], hi[None], np.array([B]))[0]
    exact = O.osa_head_masses(q[None], keys, B, B, 1.0 / math.sqrt(d))[0, 0]
    assert abs(s - exact) <= 1e-12 * abs(exact)
    assert abs(s - (math.log(B) + q @ k / math.sqrt(d))) <= 1e-12 * abs(s)


def test_group_score_is_the_log_of_summed_head_bounds():
    rng = np.random.default_rng(4)
    d = 32
    keys = rng.normal(size=(3 * 64, d))
    lo, hi = O.build_block_boxes(keys, 64, 0, 3)
    qg = rng.normal(size=(4, d))
    per = np.array([O.box_head_scores(q, lo, hi, np.full(3, 64)) for q in qg])
    want = np.log(np.exp(per).sum(axis=0))
    np.testing.assert_allclose(O.box_group_scores(qg, lo, hi, np.full(3, 64)), want,
                               rtol=1e-13)


def test_box_selection_follows_the_selection_rules():
    """Forced sink and local blocks, then the best candidates by box score."""
    rng = np.random.default_rng(5)
    d, B, L = 32, 64, 64 * 40 + 17
    keys = rng.normal(size=(L, d))
    # a block whose keys stretch far along the group's queries must win
    qg = rng.normal(size=(2, d))
    keys[20 * B:21 * B] += 4.0 * np.sign(qg.sum(axis=0))
    lo, hi = O.build_block_boxes(keys, B, 0, L // B)
    sel, scores = O.select_from_boxes(qg, lo, hi, L, B, 3, 1, 200)
    forced, c0, c1 = O.block_partition(L, B, 1, 200)
    assert set(forced) <= set(sel.tolist()) and len(sel) == len(forced) + 3
    assert 20 in sel
    cand = [j for j in sel if c0 <= j < c1]
    rest = [j for j in range(c0, c1) if j not in cand]
    assert min(scores[j] for j in cand) >= max(scores[j] for j in rest)


# ---------------------------------------------------------------------------
# plausible mistakes planted in the oracle (on the CPU) must trip a pin
# ---------------------------------------------------------------------------

def _expect_pin_failure(monkeypatch, name, bad, pin):
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        pin()


def test_mutation_box_centre_only(monkeypatch):
    def bad(q, lo, hi, n):      # the box's centre, not its reach
        return np.log(np.asarray(n, float)) + ((lo + hi) / 2) @ q / math.sqrt(len(q))
    _expect_pin_failure(monkeypatch, "box_head_scores", bad,
                        test_score_is_the_maximum_over_the_corners)


def test_mutation_box_min_instead_of_max(monkeypatch):
    def bad(q, lo, hi, n):
        reach = np.sum(np.minimum(q[None, :] * lo, q[None, :] * hi), axis=1)
        return np.log(np.asarray(n, float)) + reach / math.sqrt(len(q))
    _expect_pin_failure(monkeypatch, "box_head_scores", bad,
                        test_score_bounds_the_exact_log_mass_from_above)
