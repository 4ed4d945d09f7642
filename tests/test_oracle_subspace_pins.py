"""Pins of the oracle's subspace projection (COBS explainer §2.3: covariance
projected onto the top eigenvectors of the queries' second moment) against
what fixes it from outside the oracle: calibration queries built with a known
second moment (orthonormal directions with planted variances), so the
subspace is known in closed form; the full subspace (s = d) and queries inside
the subspace leave the score unchanged; the projected quadratic term is the
covariance's quadratic form at the projected query, by hand."""

import math

import numpy as np
import pytest

import oracle.cobs_oracle as O


def planted_queries(n, d, variances, seed):
    """Queries whose second moment is exactly V diag(variances) V^T.

    C holds columns 1..k of an n x n Sylvester Hadamard matrix (zero mean,
    (1/n) C^T C = I), placed along random orthonormal directions V."""
    rng = np.random.default_rng(seed)
    k = len(variances)
    v, _ = np.linalg.qr(rng.standard_normal((d, k)))
    # n x k with orthogonal columns of squared norm n (n a power of two >= k + 1)
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    c = h[:, 1:1 + k]
    return c @ np.diag(np.sqrt(variances)) @ v.T, v


def test_subspace_is_the_planted_top_directions():
    d, n = 32, 64
    var = np.array([9.0, 7.0, 5.0, 3.0, 1.0, 0.5])
    q_cal, v = planted_queries(n, d, var, seed=0)
    for s in (1, 3, 5):
        p = O.query_subspace(q_cal, s)
        assert p.shape == (d, s)
        np.testing.assert_allclose(p.T @ p, np.eye(s), atol=1e-12)
        # the span equals the span of the s directions of largest variance
        proj_true = v[:, :s] @ v[:, :s].T
        np.testing.assert_allclose(p @ p.T, proj_true, atol=1e-10)
        # each column is its planted direction up to sign (distinct variances)
        for j in range(s):
            assert abs(abs(p[:, j] @ v[:, j]) - 1.0) <= 1e-10


def test_full_subspace_leaves_the_score_unchanged():
    rng = np.random.default_rng(1)
    d, B = 32, 64
    keys = O.round_to_bf16(rng.normal(0.0, 0.5, size=(4 * B, d)))
    p = O.query_subspace(rng.normal(size=(200, d)), d)
    mu, us = O.build_block_records_subspace(keys, B, 4, p, 0, 4, to_bf16=False)
    rec = O.build_block_records(keys, B, 4, 0, 4, to_bf16=False)
    q = rng.normal(size=d)
    np.testing.assert_allclose(O.subspace_head_scores(q, mu, us, p, np.full(4, B)),
                               O.head_block_scores(q, rec, np.full(4, B)), rtol=1e-12)


def test_queries_inside_the_subspace_lose_nothing():
    rng = np.random.default_rng(2)
    d, B, s = 32, 64, 6
    keys = O.round_to_bf16(rng.normal(0.0, 0.5, size=(3 * B, d)))
    q_cal, v = planted_queries(64, d, np.arange(8, 0, -1.0), seed=3)
    p = O.query_subspace(q_cal, s)
    mu, us = O.build_block_records_subspace(keys, B, 8, p, 0, 3, to_bf16=False)
    rec = O.build_block_records(keys, B, 8, 0, 3, to_bf16=False)
    q = p @ rng.normal(size=s)                       # a query in span(P)
    np.testing.assert_allclose(O.subspace_head_scores(q, mu, us, p, np.full(3, B)),
                               O.head_block_scores(q, rec, np.full(3, B)), rtol=1e-12)


def test_quadratic_term_is_the_covariance_form_at_the_projected_query():
    rng = np.random.default_rng(4)
    d, B, s, r = 16, 64, 5, 4
    keys = rng.normal(size=(B, d))
    p = O.query_subspace(rng.normal(size=(100, d)), s)
    mu, us = O.block_record_subspace(keys, r, p, to_bf16=False)
    _, sigma = O.block_moments(keys)
    u, _ = O.covariance_factor(sigma, r)
    q = rng.normal(size=d)
    qp = p @ (p.T @ q)                                # projected query, by hand
    want = (math.log(B) + mu @ q / math.sqrt(d) + 0.5 * qp @ (u @ u.T) @ qp / d)
    got = O.subspace_head_scores(q, mu[None], us[None], p, np.array([B]))[0]
    assert abs(got - want) <= 1e-12 * abs(want)
    assert us.shape == (r, s)                         # r x s stored values, not r x d


def test_subspace_selection_follows_the_selection_rules():
    rng = np.random.default_rng(5)
    d, B, L = 32, 64, 64 * 30 + 5
    keys = rng.normal(size=(L, d))
    p = O.query_subspace(rng.normal(size=(300, d)), 8)
    mu, us = O.build_block_records_subspace(keys, B, 4, p, 0, L // B)
    qg = rng.normal(size=(2, d))
    sel, scores = O.select_from_subspace_records(qg, mu, us, p, L, B, 4, 1, 128)
    forced, c0, c1 = O.block_partition(L, B, 1, 128)
    assert set(forced) <= set(sel.tolist()) and len(sel) == len(forced) + 4
    cand = [j for j in sel if c0 <= j < c1]
    rest = [j for j in range(c0, c1) if j not in cand]
    assert min(scores[j] for j in cand) >= max(scores[j] for j in rest)


def test_second_moment_not_covariance():
    """The subspace comes from the uncentred second moment: a common offset of
    the calibration queries, orthogonal to the planted directions and larger
    than their spread, is the top direction (a covariance would drop it)."""
    d, n = 32, 64
    q_cal, v = planted_queries(n, d, np.array([4.0, 2.0, 1.0]), seed=6)
    rng = np.random.default_rng(7)
    m = rng.standard_normal(d)
    m -= v @ (v.T @ m)                                # orthogonal to the planted directions
    m *= 3.0 / np.linalg.norm(m)                      # |m|^2 = 9 > 4
    p = O.query_subspace(q_cal + m[None, :], 2)
    assert abs(abs(p[:, 0] @ m) / 3.0 - 1.0) <= 1e-10
    assert abs(abs(p[:, 1] @ v[:, 0]) - 1.0) <= 1e-10


# ---------------------------------------------------------------------------
# plausible mistakes planted in the oracle (on the CPU) must trip a pin
# ---------------------------------------------------------------------------

def _expect_pin_failure(monkeypatch, name, bad, pin):
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        pin()


def test_mutation_centred_covariance(monkeypatch):
    def bad(q_cal, s):
        q_cal = np.asarray(q_cal, dtype=np.float64)
        c = q_cal - q_cal.mean(axis=0)
        lam, vecs = np.linalg.eigh(c.T @ c / q_cal.shape[0])
        return vecs[:, np.argsort(-lam, kind="stable")[:s]]
    _expect_pin_failure(monkeypatch, "query_subspace", bad, test_second_moment_not_covariance)


def test_mutation_query_not_projected(monkeypatch):
    def bad(q, mu, us, p, n):   # the first s query components instead of P^T q
        q = np.asarray(q, dtype=np.float64)
        d, s = p.shape
        proj = us @ q[:s]
        return (np.log(np.asarray(n, float)) + mu @ q / math.sqrt(d)
                + 0.5 * np.sum(proj * proj, axis=1) / d)
    _expect_pin_failure(monkeypatch, "subspace_head_scores", bad,
                        test_queries_inside_the_subspace_lose_nothing)
