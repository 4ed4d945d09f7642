"""Pins for the CPU oracle: each check ties it to something other than itself.

What pins what (COBS explainer = gist.science paper 2607.09052):

* bf16 storage (§2.3 "block means in BF16"): hand-worked ties and torch's own
  fp32 -> bf16 conversion.
* Moments and eigen factor (§2.2 kappa1/kappa2, §2.3 top-r eigenpairs):
  blocks built from a Hadamard design whose empirical mean and population
  covariance are known exactly, with a planted spectrum.
* Second-order score (§2.2 cumulant expansion, §2.3 score): the exact Gaussian
  log-moment-generating function (closed form), and a Monte-Carlo estimate of
  ln E[exp(q.k/sqrt d)] from 10^6 samples.
* First-order reduction (§2.2: first-order selectors keep only the linear
  term): r = 0 equals a zeroed covariance factor and ranks by q.mu.
* Attention (glossary "LLMアテンション機構", scaled dot-product attention):
  torch's fp64 scaled_dot_product_attention; log-normaliser vs scipy.
* k = all blocks reduces sparse attention to dense attention.
* Exact block masses (§2.1 OSA) sum to the dense attention normaliser.
* Selection (top-k + sink + local window): invariants, planted ties, edge
  cases of the block partition.
* A hand-derived 2-d example (tests/golden/two_dim_block.json).
* Mutation checks: plausible mistakes planted in a copy of the oracle make the
  pins fail.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle.cobs_oracle as O
from workloads import WORKLOADS, bits_to_f64, make_kv_slice, make_queries

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# helpers that build inputs with known answers
# ---------------------------------------------------------------------------

def hadamard(n):
    h = np.array([[1.0]])
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def planted_block(n, d, lam, mu, seed=0):
    """Keys with empirical mean ``mu`` and population covariance V diag(lam) V^T.

    Columns 1..len(lam) of an n x n Hadamard matrix have zero mean and
    (1/n) C^T C = I, so K = 1 mu^T + C diag(sqrt lam) V^T has exactly those
    moments.  Returns (keys, V) with V orthonormal [d, len(lam)].
    """
    rng = np.random.default_rng(seed)
    r = len(lam)
    c = hadamard(n)[:, 1:1 + r]
    v, _ = np.linalg.qr(rng.standard_normal((d, r)))
    keys = mu[None, :] + c @ np.diag(np.sqrt(lam)) @ v.T
    return keys, v


# ---------------------------------------------------------------------------
# bf16 storage
# ---------------------------------------------------------------------------

def test_bf16_rounding_hand_cases():
    u = 2.0 ** -7
    cases = {1.0: 1.0, 1.0 + u / 2: 1.0, 1.0 + 1.5 * u: 1.0 + 2 * u,
             1.0 + 0.49 * u: 1.0, 1.0 + 0.51 * u: 1.0 + u, -3.0: -3.0,
             math.sqrt(2): 1.4140625, 0.0: 0.0}
    for x, want in cases.items():
        assert O.round_to_bf16(np.array([x]))[0] == want, x


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal(100000) * 10.0 ** rng.uniform(-3, 3, 100000))
    x = x.astype(np.float32).astype(np.float64)     # exactly fp32-representable
    want = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.round_to_bf16(x), want)


# ---------------------------------------------------------------------------
# moments and eigen factor
# ---------------------------------------------------------------------------

def test_moments_of_planted_block_are_exact():
    d, n = 16, 64
    lam = np.array([5.0, 3.0, 2.0, 0.5])
    mu = np.linspace(-1, 1, d)
    keys, v = planted_block(n, d, lam, mu)
    m, s = O.block_moments(keys)
    np.testing.assert_allclose(m, mu, atol=1e-13)
    np.testing.assert_allclose(s, v @ np.diag(lam) @ v.T, atol=1e-12)


def test_factor_reproduces_planted_covariance_and_truncates():
    d, n = 32, 64
    lam = np.array([9.0, 4.0, 2.5, 1.0, 0.25, 0.1])
    keys, v = planted_block(n, d, lam, np.zeros(d), seed=3)
    _, s = O.block_moments(keys)
    for r in (1, 3, 6, 8):
        u, lr = O.covariance_factor(s, r)
        k = min(r, len(lam))
        want = v[:, :k] @ np.diag(lam[:k]) @ v[:, :k].T
        np.testing.assert_allclose(u @ u.T, want, atol=1e-11)
        np.testing.assert_allclose(lr[:k], lam[:k], atol=1e-11)
        # columns are +-sqrt(lambda) times the planted directions, descending
        for j in range(k):
            cos = abs(u[:, j] @ v[:, j]) / np.linalg.norm(u[:, j])
            assert cos == pytest.approx(1.0, abs=1e-10)
            i = np.argmax(np.abs(u[:, j]))
            assert u[i, j] > 0


def test_record_layout_and_rounding():
    d, n = 8, 64
    lam = np.array([3.0, 1.0])
    mu = np.arange(d) / 7.0
    keys, v = planted_block(n, d, lam, mu, seed=5)
    rec = O.block_record(keys, 2)
    assert rec.shape == (3, d)
    np.testing.assert_array_equal(rec[0], O.round_to_bf16(mu))
    exact = O.block_record(keys, 2, to_bf16=False)
    np.testing.assert_array_equal(rec, O.round_to_bf16(exact))
    np.testing.assert_allclose(exact[1:].T @ exact[1:], v @ np.diag(lam) @ v.T,
                               atol=1e-12)


# ---------------------------------------------------------------------------
# second-order score
# ---------------------------------------------------------------------------

def test_score_equals_gaussian_log_mgf_closed_form():
    d, n = 32, 64
    rng = np.random.default_rng(7)
    lam = np.array([4.0, 2.0, 1.0, 0.5])
    mu = 0.3 * rng.standard_normal(d)
    keys, v = planted_block(n, d, lam, mu, seed=7)
    rec = O.block_record(keys, 4, to_bf16=False)
    sigma = v @ np.diag(lam) @ v.T
    for _ in range(5):
        q = rng.standard_normal(d)
        a = q / math.sqrt(d)
        want = math.log(n) + a @ mu + 0.5 * a @ sigma @ a
        got = O.head_block_scores(q, rec[None], np.array([n]))[0]
        assert got == pytest.approx(want, abs=1e-12)


def test_score_matches_monte_carlo_attention_mass():
    """ln E exp(q.k/sqrt d) for k ~ N(mu, Sigma): the quantity m_b/L estimates."""
    d = 16
    rng = np.random.default_rng(11)
    lam = np.array([1.5, 0.8, 0.3])
    v, _ = np.linalg.qr(rng.standard_normal((d, 3)))
    mu = 0.2 * rng.standard_normal(d)
    q = rng.standard_normal(d)
    u = v * np.sqrt(lam)
    rec = np.concatenate([mu[None], u.T])[None]
    score = O.head_block_scores(q, rec, np.array([1]))[0]      # ln 1 = 0
    z = rng.standard_normal((1_000_000, 3))
    logits = (mu + z @ u.T) @ q / math.sqrt(d)
    w = np.exp(logits)
    est = math.log(w.mean())
    se = w.std() / w.mean() / math.sqrt(len(w))
    assert abs(est - score) < 4 * se + 1e-9


def test_rank_zero_is_the_mean_only_selector():
    w = WORKLOADS["tiny_4k"]
    q = bits_to_f64(make_queries(w))[0]
    kb, _ = make_kv_slice(w, 0, 0)
    keys = bits_to_f64(kb)
    nb = w.seq_len // w.block
    rec4 = O.build_block_records(keys, w.block, 4, 0, nb)
    rec0 = O.build_block_records(keys, w.block, 0, 0, nb)
    zeroed = rec4.copy()
    zeroed[:, 1:] = 0.0
    n = np.full(nb, w.block)
    s0 = O.group_block_scores(q, rec0, n)
    np.testing.assert_array_equal(s0, O.group_block_scores(q, zeroed, n))
    # first-order score: ranking of blocks follows ln sum_h exp(q_h.mu/sqrt d)
    lin = scipy.special.logsumexp(q @ rec0[:, 0].T / math.sqrt(w.head_dim), axis=0)
    np.testing.assert_array_equal(np.argsort(-s0, kind="stable"),
                                  np.argsort(-lin, kind="stable"))


def test_wider_block_ranks_higher_for_aligned_query():
    """§ "the problem": two blocks with the same mean, the wider one holds more
    mass along the query; the first-order score cannot tell them apart."""
    d, n = 16, 64
    q = np.zeros(d)
    q[0] = 4.0
    mu = np.zeros(d)
    direc = np.eye(d)[:, :1]
    tight = mu + hadamard(n)[:, 1:2] @ direc.T * 0.3
    wide = mu + hadamard(n)[:, 1:2] @ direc.T * 2.0
    recs = np.stack([O.block_record(tight, 2, False), O.block_record(wide, 2, False)])
    s = O.head_block_scores(q, recs, np.array([n, n]))
    assert s[1] > s[0]
    s_first = O.head_block_scores(q, recs[:, :1], np.array([n, n]))
    assert s_first[0] == s_first[1]
    masses = O.osa_head_masses(q[None], np.concatenate([tight, wide]), 2 * n, n,
                               1 / math.sqrt(d))[0]
    assert masses[1] > masses[0]


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def _rand_attention_case(rng, g=4, t=300, d=32):
    return (rng.standard_normal((g, d)), rng.standard_normal((t, d)),
            rng.standard_normal((t, d)))


def test_dense_attention_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(2)
    for t in (1, 7, 300):
        q, k, v = _rand_attention_case(rng, t=t)
        out, lse = O.dense_attention(q, k, v, t, 1 / math.sqrt(32))
        tq = torch.from_numpy(q)[None, :, None, :]
        tk = torch.from_numpy(k)[None, None].expand(1, 4, t, 32)
        tv = torch.from_numpy(v)[None, None].expand(1, 4, t, 32)
        want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)
        np.testing.assert_allclose(out, want[0, :, 0].numpy(), atol=1e-13)
        np.testing.assert_allclose(
            lse, scipy.special.logsumexp(q @ k.T / math.sqrt(32), axis=1),
            atol=1e-12)


def test_sparse_with_all_blocks_is_dense():
    w = WORKLOADS["tiny_4k"].scaled(seq_len=1000)     # ragged tail
    q = bits_to_f64(make_queries(w))[0]
    kb, vb = make_kv_slice(w, 0, 0)
    k, v = bits_to_f64(kb), bits_to_f64(vb)
    recs = O.build_block_records(k, w.block, w.rank, 0, w.seq_len // w.block)
    sel, _, out, lse = O.decode_step(q, k, v, recs, w.seq_len, w.block,
                                     top_k=10 ** 6, sink_blocks=1,
                                     local_tokens=64)
    assert list(sel) == list(range(-(-w.seq_len // w.block)))
    dout, dlse = O.dense_attention(q, k, v, w.seq_len, 1 / math.sqrt(w.head_dim))
    np.testing.assert_allclose(out, dout, atol=1e-12)
    np.testing.assert_allclose(lse, dlse, atol=1e-12)


def test_exact_block_masses_sum_to_dense_normaliser():
    rng = np.random.default_rng(4)
    q, k, v = _rand_attention_case(rng, t=1000)
    scale = 1 / math.sqrt(32)
    heads = O.osa_head_masses(q, k, 1000, 64, scale)
    _, lse = O.dense_attention(q, k, v, 1000, scale)
    np.testing.assert_allclose(scipy.special.logsumexp(heads, axis=1), lse,
                               atol=1e-12)
    group = O.osa_group_masses(q, k, 1000, 64, scale)
    np.testing.assert_allclose(scipy.special.logsumexp(group),
                               scipy.special.logsumexp(lse), atol=1e-12)


# ---------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,B,sink,W,forced,c0,c1", [
    (4096, 64, 1, 64, [0, 63], 1, 63),
    (4096, 64, 1, 512, [0] + list(range(56, 64)), 1, 56),
    (1000, 64, 1, 64, [0, 14, 15], 1, 14),          # T-W=936 -> block 14
    (1000, 64, 1, 0, [0, 15], 1, 15),               # partial tail is forced
    (1024, 64, 1, 0, [0], 1, 16),                   # no local block at all
    (300, 64, 1, 512, [0, 1, 2, 3, 4], 0, 0),       # window covers everything
    (130, 64, 3, 10, [0, 1, 2], 1, 1),              # sink overlaps local
    (64, 64, 1, 1, [0], 0, 0),
])
def test_block_partition_cases(T, B, sink, W, forced, c0, c1):
    f, a, b = O.block_partition(T, B, sink, W)
    assert (f, a, b) == (forced, c0, c1)


def test_selection_invariants_and_ties():
    rng = np.random.default_rng(9)
    T, B, k = 64 * 40 + 17, 64, 7
    scores = rng.standard_normal(T // B)
    scores[[5, 9, 13, 22]] = 30.0                # four-way tie at the top...
    scores[[30, 31]] = 25.0
    sel = O.select_blocks(scores, T, B, k, 1, 100)
    forced, c0, c1 = O.block_partition(T, B, 1, 100)
    assert np.all(np.diff(sel) > 0)
    assert set(forced) <= set(sel)
    chosen = [j for j in sel if j not in forced]
    assert len(chosen) == k
    rest = [j for j in range(c0, c1) if j not in chosen]
    assert min(scores[chosen]) >= max(scores[rest])
    assert {5, 9, 13, 22, 30, 31} <= set(chosen)
    # tie at the boundary: the lower indices win
    scores2 = np.zeros(T // B)
    sel2 = O.select_blocks(scores2, T, B, 3, 1, 100)
    assert [j for j in sel2 if j not in forced] == [1, 2, 3]


def test_top_k_at_least_candidates_takes_everything():
    sel = O.select_blocks(np.zeros(10), 640, 64, 50, 1, 64)
    assert list(sel) == list(range(10))


def test_selection_by_exact_mass_recovers_needles():
    """On the needle recipe, oracle sparse attention (§2.1) must find the
    planted blocks, and the second-order score should find at least as many
    as the first-order one (§2.2-2.3)."""
    w = WORKLOADS["batched_needles_32k"].scaled(batch=2, seq_len=8192)
    qb = make_queries(w)
    scale = 1 / math.sqrt(w.head_dim)
    nb = w.seq_len // w.block
    hits = {"osa": 0, "cobs": 0, "mean": 0}
    total = 0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            kb, vb = make_kv_slice(w, b, h, qb)
            k = bits_to_f64(kb)
            qg = bits_to_f64(qb[b, h * w.group:(h + 1) * w.group])
            # needle blocks: the planted tokens point along the group's mean
            # query (cosine 0.9); ordinary keys are nearly orthogonal to it
            qhat = qg.mean(axis=0) / np.linalg.norm(qg.mean(axis=0))
            cos = (k[:w.seq_len] @ qhat) / np.linalg.norm(k[:w.seq_len], axis=1)
            needles = set(np.unique(np.nonzero(cos > 0.8)[0] // w.block))
            needles = {j for j in needles if 1 <= j < nb - 8}
            total += len(needles)
            osa = O.osa_group_masses(qg, k, w.seq_len, w.block, scale)
            recs = O.build_block_records(k, w.block, w.rank, 0, nb)
            for name, r in (("cobs", recs), ("mean", recs[:, :1])):
                sel, _ = O.select_from_records(qg, r, w.seq_len, w.block,
                                               w.top_k, 1, w.local_tokens)
                hits[name] += len(needles & set(sel.tolist()))
            sel = O.select_blocks(osa, w.seq_len, w.block, w.top_k, 1,
                                  w.local_tokens)
            hits["osa"] += len(needles & set(sel.tolist()))
    assert total >= 4 * w.batch * w.kv_heads * 0.9
    assert hits["osa"] == total
    assert hits["cobs"] > hits["mean"]


# ---------------------------------------------------------------------------
# hand-derived golden example
# ---------------------------------------------------------------------------

def test_two_dim_golden_block():
    g = json.load(open(os.path.join(GOLDEN, "two_dim_block.json")))
    keys = np.array(g["keys"], dtype=float)
    q = np.array(g["query"], dtype=float)
    mu, sigma = O.block_moments(keys)
    np.testing.assert_allclose(mu, g["mean"], atol=0)
    np.testing.assert_allclose(sigma, g["covariance_population"], atol=1e-15)
    u, lam = O.covariance_factor(sigma, 2)
    np.testing.assert_allclose(lam, g["eigenvalues_desc"], atol=1e-14)
    np.testing.assert_allclose(u.T, g["U_columns_rank2"], atol=1e-14)
    rec1 = O.block_record(keys, 1)
    np.testing.assert_array_equal(rec1, np.array(g["record_rank1_bf16"]))
    ln4 = math.log(4)
    full = np.concatenate([mu[None], O.covariance_factor(sigma, 2)[0].T])[None]
    assert O.head_block_scores(q, full, [4])[0] - ln4 == pytest.approx(
        g["score_full_cov_minus_ln4"], abs=1e-14)
    exact1 = O.block_record(keys, 1, to_bf16=False)[None]
    assert O.head_block_scores(q, exact1, [4])[0] - ln4 == pytest.approx(
        g["score_rank1_exact_minus_ln4"], abs=1e-14)
    assert O.head_block_scores(q, rec1[None], [4])[0] - ln4 == pytest.approx(
        g["score_rank1_bf16_record_minus_ln4"], abs=1e-15)
    r2 = math.sqrt(2)
    mass = O.osa_head_masses(q[None], keys, 4, 4, 1 / r2)[0, 0]
    assert mass == pytest.approx(math.log(2 * math.cosh(r2) + 2 * math.cosh(2 * r2)),
                                 abs=1e-14)


# ---------------------------------------------------------------------------
# mutation checks: plausible mistakes must trip a pin
# ---------------------------------------------------------------------------

def _expect_pin_failure(monkeypatch, name, bad, pin):
    monkeypatch.setattr(O, name, bad)
    with pytest.raises(AssertionError):
        pin()


def test_mutation_sample_covariance(monkeypatch):
    def bad_moments(keys):
        keys = np.asarray(keys, float)
        mu = keys.mean(0)
        c = keys - mu
        return mu, c.T @ c / (keys.shape[0] - 1)
    _expect_pin_failure(monkeypatch, "block_moments", bad_moments,
                        test_moments_of_planted_block_are_exact)


def test_mutation_score_missing_half(monkeypatch):
    def bad(q, records, n):
        d = len(q)
        p = records[:, 1:, :] @ q
        return (np.log(np.asarray(n, float)) + records[:, 0, :] @ q / math.sqrt(d)
                + np.sum(p * p, 1) / d)
    _expect_pin_failure(monkeypatch, "head_block_scores", bad,
                        test_score_equals_gaussian_log_mgf_closed_form)


def test_mutation_score_unscaled_linear_term(monkeypatch):
    def bad(q, records, n):
        d = len(q)
        p = records[:, 1:, :] @ q
        return (np.log(np.asarray(n, float)) + records[:, 0, :] @ q
                + 0.5 * np.sum(p * p, 1) / d)
    _expect_pin_failure(monkeypatch, "head_block_scores", bad,
                        test_score_matches_monte_carlo_attention_mass)


def test_mutation_factor_without_sqrt(monkeypatch):
    orig = O.covariance_factor

    def bad(sigma, rank):
        u, lam = orig(sigma, rank)
        nrm = np.linalg.norm(u, axis=0)
        nrm[nrm == 0] = 1
        return u / nrm * lam, lam
    _expect_pin_failure(monkeypatch, "covariance_factor", bad,
                        test_factor_reproduces_planted_covariance_and_truncates)


def test_mutation_tie_break_reversed(monkeypatch):
    def bad(scores, seq_len, block, top_k, sink_blocks, local_tokens):
        forced, c0, c1 = O.block_partition(seq_len, block, sink_blocks,
                                           local_tokens)
        cand = np.arange(c0, c1)
        s = np.asarray(scores, float)[c0:c1]
        order = np.lexsort((-cand, -s))
        return np.sort(np.concatenate([np.asarray(forced, int), cand[order[:top_k]]]))
    _expect_pin_failure(monkeypatch, "select_blocks", bad,
                        test_selection_invariants_and_ties)


def test_mutation_attention_wrong_scale(monkeypatch):
    orig = O.softmax_attention

    def bad(q, k, v, scale):
        return orig(q, k, v, scale * math.sqrt(2))
    _expect_pin_failure(monkeypatch, "softmax_attention", bad,
                        test_dense_attention_matches_torch_sdpa_fp64)
