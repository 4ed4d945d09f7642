"""Plain fp64 CPU oracle for COBS block-sparse attention decode.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the tests, the smoke check of
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
module.  It shares no code with the CUDA library (no kernels, headers, helpers,
tables or constants) and never imports it; the only thing both sides see is the
seeded input generator in ``workloads/``.

Everything here is written for a reader who wants to check it against the
sources by eye: numpy fp64 throughout, library primitives (matmul, eigh, sort)
as single steps, no blocking, fusion or reordering beyond what the method
itself states.  Inputs arrive as the exact bf16 values widened to fp64.

Sources (the pages the method is described on):

* "COBS: Cumulant Order Block Sparse Attention" (AI-generated explainer,
  gist.science paper 2607.09052), technical summary:
    - §2.1 selection oracle: a block's attention mass m_b is the sum of
      exp(q.k) over its keys; ranking blocks by m_b is the optimal criterion
      and "oracle sparse attention" (OSA) ranks by the exact mass.
    - §2.2 cumulant expansion: ln m_b = ln L + q.kappa1 + 1/2 q^T kappa2 q + ...
      with kappa1 the block's mean key and kappa2 its key covariance.
    - §2.3 COBS: score_b ~ q.mean_b + 1/2 q^T Sigma_b q; the covariance is kept
      as its top-r eigenvectors and eigenvalues; block means are stored in bf16.
* "LLMアテンション機構" (jisaku.com glossary), section on the computing
  principle of self-attention: softmax(q K^T / sqrt(d_k)) V; GQA shares one
  K/V head between several query heads; the KV cache keeps K and V per token.
* "スライディングウィンドウアテンション" (jisaku.com glossary), overview and
  extensions: a local window of the last w tokens; attention-sink tokens at the
  start of the sequence are always kept.

Readings taken where the pages are silent or garbled (each also listed in the
design notes of the repository):

* The score uses the attention logit scale: a = q / sqrt(d), so
  score_b = ln n_b + a.mu_b + 1/2 a^T Sigma_b a
          = ln n_b + (q.mu_b)/sqrt(d) + 1/2 ||U_b^T q||^2 / d.
  The pages' formula for the score omits both 1/sqrt(d) and ln L; ln n_b is
  kept (it is constant over the complete blocks that compete in top-k).
* Sigma_b is the population covariance (1/n) sum (k - mu)(k - mu)^T: the
  second cumulant of the block's empirical key distribution.
* U_b = V_r Lambda_r^{1/2} (top-r eigenpairs, descending eigenvalue), each
  column's sign fixed so that its largest-magnitude component is positive
  (the score does not depend on the sign; this only makes dumps
  deterministic).  The stored record is [mu; U columns as rows] rounded to bf16.
* One selection per (batch, kv-head): the group score is the log of the
  group's total estimated mass, S_b = ln sum_h exp(s_{h,b}).
* Forced blocks: the first ``sink_blocks`` blocks (attention sink) and every
  block that intersects the last ``local_tokens`` tokens, plus the partial
  tail block (which has no statistics).  Top-k runs over the remaining
  complete blocks; ties go to the lower block index.  Output ascending.
* Attention over the selected blocks is one exact softmax over the union of
  their valid tokens, with the 1/sqrt(d) logit scale.
* Subspace projection (§2.3): the covariance is projected onto the span P
  (d x s, orthonormal columns) of the top s eigenvectors of the queries'
  second moment M = (1/n) sum q q^T over a set of calibration queries, so a
  block stores U_s = P^T U (r x s values instead of r x d); the score's
  quadratic term becomes 1/2 |U_s^T P^T q|^2 / d = 1/2 (P P^T q)^T Sigma_r
  (P P^T q) / d.  The mean and the linear term keep all d dimensions.
* The min/max box selector (explainer, plain-language summary of what the
  paper rules out: the spread of a block estimated from the minimum and
  maximum of its keys; it helps somewhat, less than COBS; no formula is
  given): the box is the per-dimension minimum lo and maximum hi of the
  block's keys, and a block's score is ln n_b plus the largest logit any
  point of the box can reach, max_{lo <= k <= hi} q.k / sqrt(d) =
  sum_t max(q_t lo_t, q_t hi_t) / sqrt(d) -- an upper bound of the block's
  log attention mass.  Groups aggregate as for COBS.
* FP4 storage of U (§2.3, quantisation: eigenvectors stored scaled in FP4
  E2M1, block means in BF16): every U column is cut into groups of 32
  consecutive components; each group stores E2M1 codes and one power-of-two
  scale 2^e (an 8-bit biased exponent, as in the E8M0 scales of the OCP
  microscaling formats), e being the smallest exponent with
  max |u| <= 6 * 2^e, so that no component saturates; components are rounded
  to the nearest E2M1 value, ties to the even code.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "round_to_bf16",
    "block_moments",
    "covariance_factor",
    "block_record",
    "build_block_records",
    "head_block_scores",
    "group_block_scores",
    "block_partition",
    "select_blocks",
    "select_from_records",
    "tokens_of_blocks",
    "softmax_attention",
    "sparse_attention",
    "dense_attention",
    "osa_head_masses",
    "osa_group_masses",
    "decode_step",
    "E2M1_MAGNITUDES",
    "FP4_GROUP",
    "e2m1_value",
    "round_to_e2m1",
    "fp4_scale_exponent",
    "quantize_u_fp4",
    "dequantize_u_fp4",
    "block_record_fp4",
    "build_block_records_fp4",
    "fp4_record_values",
    "block_box",
    "build_block_boxes",
    "box_head_scores",
    "box_group_scores",
    "select_from_boxes",
    "query_subspace",
    "project_factor",
    "block_record_subspace",
    "build_block_records_subspace",
    "subspace_head_scores",
    "subspace_group_scores",
    "select_from_subspace_records",
]


# ---------------------------------------------------------------------------
# bf16 storage (COBS explainer §2.3: block means are stored in BF16; the same
# record format holds the covariance factor in this build)
# ---------------------------------------------------------------------------

def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), as fp64.

    bf16 keeps 8 significant bits (7 stored), so on the fp64 bit pattern the
    low 52 - 7 = 45 mantissa bits are rounded away in one step (no fp32
    intermediate, hence no double rounding).  Valid for finite values inside
    the bf16 normal range, which is all this oracle stores.
    """
    x64 = np.ascontiguousarray(x, dtype=np.float64)
    u = x64.view(np.uint64)
    drop = np.uint64(45)
    lsb = (u >> drop) & np.uint64(1)
    half = np.uint64((1 << 44) - 1)
    mask = ~np.uint64((1 << 45) - 1)
    r = ((u + half + lsb) & mask).view(np.float64)
    return np.where(x64 == 0.0, x64, r)


# ---------------------------------------------------------------------------
# Block statistics (COBS explainer §2.2 cumulants, §2.3 low-rank factor)
# ---------------------------------------------------------------------------

def block_moments(keys: np.ndarray):
    """First and second cumulants of one block's keys.

    kappa1 = mean key; kappa2 = population covariance (1/n) sum (k-mu)(k-mu)^T,
    computed two-pass (mean first, then centred products).
    """
    keys = np.asarray(keys, dtype=np.float64)
    n = keys.shape[0]
    mu = keys.sum(axis=0) / n
    centred = keys - mu
    sigma = centred.T @ centred / n
    return mu, sigma


def covariance_factor(sigma: np.ndarray, rank: int):
    """Top-``rank`` eigenpairs of a covariance as a factor U with U U^T = Sigma_r.

    COBS explainer §2.3 (low-rank factorisation): keep the top r eigenvectors
    and eigenvalues.  Returns (U [d, r], eigenvalues [r], descending).
    """
    d = sigma.shape[0]
    if rank == 0:
        return np.zeros((d, 0)), np.zeros(0)
    lam, vecs = np.linalg.eigh(sigma)
    order = np.argsort(-lam, kind="stable")[:rank]
    lam_r = np.clip(lam[order], 0.0, None)
    v_r = vecs[:, order]
    for j in range(v_r.shape[1]):
        i = int(np.argmax(np.abs(v_r[:, j])))
        if v_r[i, j] < 0:
            v_r[:, j] = -v_r[:, j]
    return v_r * np.sqrt(lam_r)[None, :], lam_r


def block_record(keys: np.ndarray, rank: int, to_bf16: bool = True) -> np.ndarray:
    """The stored statistics record of one complete block: [mu; U^T], (1+r, d).

    With ``to_bf16`` (the storage format) every value is rounded to bf16.
    """
    mu, sigma = block_moments(keys)
    u, _ = covariance_factor(sigma, rank)
    rec = np.concatenate([mu[None, :], u.T], axis=0)
    return round_to_bf16(rec) if to_bf16 else rec


def build_block_records(keys_seq: np.ndarray, block: int, rank: int,
                        block_begin: int, block_end: int,
                        to_bf16: bool = True) -> np.ndarray:
    """Records for complete blocks [block_begin, block_end) of one (b, kv-head)."""
    recs = [block_record(keys_seq[j * block:(j + 1) * block], rank, to_bf16)
            for j in range(block_begin, block_end)]
    d = keys_seq.shape[1]
    if not recs:
        return np.zeros((0, 1 + rank, d))
    return np.stack(recs, axis=0)


# ---------------------------------------------------------------------------
# Scores (COBS explainer §2.2 expansion, §2.3 second-order score)
# ---------------------------------------------------------------------------

def head_block_scores(q: np.ndarray, records: np.ndarray,
                      n_tokens: np.ndarray) -> np.ndarray:
    """s_b = ln n_b + (q.mu_b)/sqrt(d) + 1/2 sum_j (u_j.q)^2 / d for every block.

    ``records``: [nb, 1+r, d]; row 0 is mu, rows 1..r are the columns of U.
    With r = 0 this is the first-order (mean-only) score.
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    linear = records[:, 0, :] @ q / math.sqrt(d)
    proj = records[:, 1:, :] @ q                       # [nb, r]
    quadratic = 0.5 * np.sum(proj * proj, axis=1) / d
    return np.log(np.asarray(n_tokens, dtype=np.float64)) + linear + quadratic


def _logsumexp(x: np.ndarray, axis: int) -> np.ndarray:
    m = np.max(x, axis=axis, keepdims=True)
    return (m + np.log(np.sum(np.exp(x - m), axis=axis, keepdims=True))).squeeze(axis)


def group_block_scores(q_group: np.ndarray, records: np.ndarray,
                       n_tokens: np.ndarray) -> np.ndarray:
    """S_b = ln sum_h exp(s_{h,b}) over the G query heads of one kv-head."""
    per_head = np.stack([head_block_scores(q, records, n_tokens)
                         for q in np.asarray(q_group, dtype=np.float64)], axis=0)
    return _logsumexp(per_head, axis=0)


# ---------------------------------------------------------------------------
# Selection: top-k + sink + local window
# ---------------------------------------------------------------------------

def block_partition(seq_len: int, block: int, sink_blocks: int,
                    local_tokens: int):
    """Split the blocks of a sequence into forced blocks and top-k candidates.

    Returns (forced_sorted, candidate_begin, candidate_end): candidates are the
    complete blocks in [candidate_begin, candidate_end).
    """
    n_blocks = -(-seq_len // block)
    n_full = seq_len // block
    first_local = min(n_full, max(0, seq_len - local_tokens) // block)
    sink_end = min(sink_blocks, first_local)
    forced = list(range(sink_end)) + list(range(first_local, n_blocks))
    return forced, sink_end, first_local


def select_blocks(scores: np.ndarray, seq_len: int, block: int, top_k: int,
                  sink_blocks: int, local_tokens: int) -> np.ndarray:
    """Top-k candidates by score (ties -> lower index), union forced, ascending.

    ``scores`` is indexed by block number; only candidate entries are read.
    """
    forced, c0, c1 = block_partition(seq_len, block, sink_blocks, local_tokens)
    cand = np.arange(c0, c1)
    s = np.asarray(scores, dtype=np.float64)[c0:c1]
    order = np.lexsort((cand, -s))            # primary: score desc; then index asc
    chosen = cand[order[:top_k]]
    return np.sort(np.concatenate([np.asarray(forced, dtype=np.int64),
                                   chosen.astype(np.int64)]))


def select_from_records(q_group, records, seq_len, block, top_k, sink_blocks,
                        local_tokens):
    """Score every complete block from its stored record, then select.

    Returns (selected indices, group scores over complete blocks).
    """
    n_full = seq_len // block
    recs = records[:n_full]
    scores = group_block_scores(q_group, recs, np.full(n_full, block))
    return select_blocks(scores, seq_len, block, top_k, sink_blocks,
                         local_tokens), scores


# ---------------------------------------------------------------------------
# Attention (glossary "LLMアテンション機構": scaled dot-product attention)
# ---------------------------------------------------------------------------

def tokens_of_blocks(blocks, seq_len: int, block: int) -> np.ndarray:
    """Valid token positions of the given blocks, in block order."""
    parts = [np.arange(j * block, min((j + 1) * block, seq_len)) for j in blocks]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def softmax_attention(q_group: np.ndarray, keys: np.ndarray, values: np.ndarray,
                      scale: float):
    """softmax(q K^T * scale) V for each head; also ln sum exp(logits)."""
    q_group = np.asarray(q_group, dtype=np.float64)
    logits = q_group @ keys.T * scale                  # [G, n]
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    l = w.sum(axis=1, keepdims=True)
    out = (w @ values) / l
    lse = (m + np.log(l))[:, 0]
    return out, lse


def sparse_attention(q_group, keys_seq, values_seq, blocks, seq_len, block,
                     scale):
    """Exact attention restricted to the valid tokens of the selected blocks."""
    t = tokens_of_blocks(blocks, seq_len, block)
    return softmax_attention(q_group, keys_seq[t], values_seq[t], scale)


def dense_attention(q_group, keys_seq, values_seq, seq_len, scale):
    """Exact attention over all ``seq_len`` cached tokens."""
    return softmax_attention(q_group, keys_seq[:seq_len], values_seq[:seq_len],
                             scale)


# ---------------------------------------------------------------------------
# Oracle sparse attention (COBS explainer §2.1): exact block masses
# ---------------------------------------------------------------------------

def osa_head_masses(q_group, keys_seq, seq_len, block, scale) -> np.ndarray:
    """ln m_b per head and block: ln sum_{t in b} exp(q_h.k_t * scale), [G, nb]."""
    q_group = np.asarray(q_group, dtype=np.float64)
    n_blocks = -(-seq_len // block)
    logits = q_group @ keys_seq[:seq_len].T * scale
    out = np.empty((q_group.shape[0], n_blocks))
    for j in range(n_blocks):
        out[:, j] = _logsumexp(logits[:, j * block:min((j + 1) * block, seq_len)],
                               axis=1)
    return out


def osa_group_masses(q_group, keys_seq, seq_len, block, scale) -> np.ndarray:
    """ln of the group's total exact mass per block: ln sum_h m_b^(h)."""
    return _logsumexp(osa_head_masses(q_group, keys_seq, seq_len, block, scale),
                      axis=0)


# ---------------------------------------------------------------------------
# One decode step for one (batch, kv-head) pair
# ---------------------------------------------------------------------------

def decode_step(q_group, keys_seq, values_seq, records, seq_len, block, top_k,
                sink_blocks, local_tokens, scale=None):
    """Select from stored records, then attend exactly over the selection.

    Returns (selected blocks, group scores, out [G, d], lse [G]).
    """
    d = keys_seq.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    sel, scores = select_from_records(q_group, records, seq_len, block, top_k,
                                      sink_blocks, local_tokens)
    out, lse = sparse_attention(q_group, keys_seq, values_seq, sel, seq_len,
                                block, scale)
    return sel, scores, out, lse


# ---------------------------------------------------------------------------
# FP4 (E2M1) scaled storage of U (COBS explainer §2.3, quantisation: the
# eigenvectors are kept in FP4 E2M1 with a scale, the block means in BF16)
# ---------------------------------------------------------------------------

# magnitudes of the E2M1 codes 0..7 (bit 3 of a code is the sign)
E2M1_MAGNITUDES = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)
FP4_GROUP = 32          # consecutive components of a U column sharing one scale


def e2m1_value(codes) -> np.ndarray:
    """Values of E2M1 codes (4-bit: sign bit 3, magnitude index bits 0-2)."""
    codes = np.asarray(codes, dtype=np.int64)
    mag = np.asarray(E2M1_MAGNITUDES)[codes & 7]
    return np.where(codes & 8, -mag, mag)


def round_to_e2m1(x) -> np.ndarray:
    """Codes of the E2M1 values nearest to x (ties to the even code).

    Magnitudes above 6 saturate to 6; a value that rounds to zero gets the
    positive zero code.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), 6.0)
    grid = np.asarray(E2M1_MAGNITUDES)
    idx = np.arange(len(grid))
    dist = np.abs(a[..., None] - grid)
    nearest = dist == dist.min(axis=-1, keepdims=True)   # one code, or two on a tie
    even = nearest & (idx % 2 == 0)
    pick = np.where(even.any(axis=-1), np.argmax(even, axis=-1),
                    np.argmax(nearest, axis=-1))
    return np.where((x < 0) & (pick != 0), pick | 8, pick).astype(np.uint8)


def fp4_scale_exponent(amax: float):
    """Smallest integer e with amax <= 6 * 2^e, clamped below at -126.

    None for amax == 0 (a group of zeros: scale byte 0, all codes 0).
    """
    if amax == 0.0:
        return None
    _, ex = math.frexp(amax)          # amax < 2^ex
    e = ex - 4                        # amax >= 2^(ex-1) > 6 * 2^(ex-4)
    while amax > 6.0 * 2.0 ** e:
        e += 1
    return max(e, -126)


def quantize_u_fp4(u_rows: np.ndarray):
    """E2M1 codes [r, d] and biased scale exponents [r, d/32] of U's columns.

    ``u_rows``: [r, d], row j = column j of U.  Scale byte = e + 127.
    """
    u_rows = np.asarray(u_rows, dtype=np.float64)
    r, d = u_rows.shape
    codes = np.zeros((r, d), dtype=np.uint8)
    scale_bytes = np.zeros((r, d // FP4_GROUP), dtype=np.uint8)
    for j in range(r):
        for g in range(d // FP4_GROUP):
            seg = u_rows[j, g * FP4_GROUP:(g + 1) * FP4_GROUP]
            e = fp4_scale_exponent(float(np.max(np.abs(seg))))
            if e is None:
                continue
            scale_bytes[j, g] = e + 127
            codes[j, g * FP4_GROUP:(g + 1) * FP4_GROUP] = round_to_e2m1(seg / 2.0 ** e)
    return codes, scale_bytes


def dequantize_u_fp4(codes, scale_bytes) -> np.ndarray:
    """Component values 2^(byte - 127) * e2m1(code); a zero scale byte is 0."""
    sb = np.asarray(scale_bytes, dtype=np.int64)
    scale = np.where(sb == 0, 0.0, np.exp2((sb - 127).astype(np.float64)))
    return e2m1_value(codes) * np.repeat(scale, FP4_GROUP, axis=-1)


def block_record_fp4(keys: np.ndarray, rank: int):
    """FP4 record of one complete block: (mu in bf16 [d], codes [r, d], scale bytes [r, d/32])."""
    mu, sigma = block_moments(keys)
    u, _ = covariance_factor(sigma, rank)
    codes, scale_bytes = quantize_u_fp4(u.T)
    return round_to_bf16(mu), codes, scale_bytes


def build_block_records_fp4(keys_seq: np.ndarray, block: int, rank: int,
                            block_begin: int, block_end: int):
    """FP4 records of complete blocks [block_begin, block_end): stacked (mu, codes, scales)."""
    d = keys_seq.shape[1]
    parts = [block_record_fp4(keys_seq[j * block:(j + 1) * block], rank)
             for j in range(block_begin, block_end)]
    if not parts:
        return (np.zeros((0, d)), np.zeros((0, rank, d), np.uint8),
                np.zeros((0, rank, d // FP4_GROUP), np.uint8))
    return tuple(np.stack(x, axis=0) for x in zip(*parts))


def fp4_record_values(mu, codes, scale_bytes) -> np.ndarray:
    """The [nb, 1+r, d] records (mu; dequantised U columns) that the score reads."""
    mu = np.asarray(mu, dtype=np.float64)
    u = dequantize_u_fp4(codes, scale_bytes)
    return np.concatenate([mu[:, None, :], u], axis=1)


# ---------------------------------------------------------------------------
# Min/max box selector (a comparison selector the explainer mentions: the
# spread of a block from the minimum and maximum of its keys)
# ---------------------------------------------------------------------------

def block_box(keys: np.ndarray):
    """Per-dimension minimum and maximum of one block's keys: (lo [d], hi [d])."""
    keys = np.asarray(keys, dtype=np.float64)
    return keys.min(axis=0), keys.max(axis=0)


def build_block_boxes(keys_seq: np.ndarray, block: int, block_begin: int, block_end: int):
    """Boxes of complete blocks [block_begin, block_end): (lo [nb, d], hi [nb, d])."""
    d = keys_seq.shape[1]
    boxes = [block_box(keys_seq[j * block:(j + 1) * block])
             for j in range(block_begin, block_end)]
    if not boxes:
        return np.zeros((0, d)), np.zeros((0, d))
    lo, hi = zip(*boxes)
    return np.stack(lo), np.stack(hi)


def box_head_scores(q: np.ndarray, lo: np.ndarray, hi: np.ndarray,
                    n_tokens: np.ndarray) -> np.ndarray:
    """s_b = ln n_b + max over the box of q.k / sqrt(d), for every block.

    The maximum of a linear function over a box is reached at a corner: in
    each dimension the end that q_t favours, so it is sum_t max(q_t lo_t,
    q_t hi_t).
    """
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    reach = np.sum(np.maximum(q[None, :] * lo, q[None, :] * hi), axis=1)
    return np.log(np.asarray(n_tokens, dtype=np.float64)) + reach / math.sqrt(d)


def box_group_scores(q_group: np.ndarray, lo: np.ndarray, hi: np.ndarray,
                     n_tokens: np.ndarray) -> np.ndarray:
    """S_b = ln sum_h exp(s_{h,b}) over the G query heads of one kv-head."""
    per_head = np.stack([box_head_scores(q, lo, hi, n_tokens)
                         for q in np.asarray(q_group, dtype=np.float64)], axis=0)
    return _logsumexp(per_head, axis=0)


def select_from_boxes(q_group, lo, hi, seq_len, block, top_k, sink_blocks, local_tokens):
    """Score every complete block by its box, then select (top-k + sink + local).

    Returns (selected indices, group scores over complete blocks).
    """
    n_full = seq_len // block
    scores = box_group_scores(q_group, lo[:n_full], hi[:n_full], np.full(n_full, block))
    return select_blocks(scores, seq_len, block, top_k, sink_blocks,
                         local_tokens), scores


# ---------------------------------------------------------------------------
# Subspace projection (COBS explainer §2.3: the covariance projected onto the
# query subspace spanned by the top eigenvectors of the queries' second
# moment, storage r x d -> r x s)
# ---------------------------------------------------------------------------

def query_subspace(q_cal: np.ndarray, s: int) -> np.ndarray:
    """P [d, s]: the top-s eigenvectors of M = (1/n) sum_i q_i q_i^T, descending
    eigenvalue, each column's largest-magnitude component made positive."""
    q_cal = np.asarray(q_cal, dtype=np.float64)
    m = q_cal.T @ q_cal / q_cal.shape[0]
    lam, vecs = np.linalg.eigh(m)
    order = np.argsort(-lam, kind="stable")[:s]
    p = vecs[:, order].copy()
    for j in range(p.shape[1]):
        i = int(np.argmax(np.abs(p[:, j])))
        if p[i, j] < 0:
            p[:, j] = -p[:, j]
    return p


def project_factor(u: np.ndarray, p: np.ndarray) -> np.ndarray:
    """U_s = P^T U: the factor's columns in subspace coordinates, [s, r]."""
    return np.asarray(p, dtype=np.float64).T @ np.asarray(u, dtype=np.float64)


def block_record_subspace(keys: np.ndarray, rank: int, p: np.ndarray,
                          to_bf16: bool = True) -> np.ndarray:
    """(mu [d], U_s^T [r, s]) of one complete block, rounded to bf16 by default."""
    mu, sigma = block_moments(keys)
    u, _ = covariance_factor(sigma, rank)
    us = project_factor(u, p).T
    if to_bf16:
        return round_to_bf16(mu), round_to_bf16(us)
    return mu, us


def build_block_records_subspace(keys_seq, block, rank, p, block_begin, block_end,
                                 to_bf16: bool = True):
    """Subspace records of complete blocks [block_begin, block_end): (mu [nb, d], us [nb, r, s])."""
    d, s = p.shape
    parts = [block_record_subspace(keys_seq[j * block:(j + 1) * block], rank, p, to_bf16)
             for j in range(block_begin, block_end)]
    if not parts:
        return np.zeros((0, d)), np.zeros((0, rank, s))
    mu, us = zip(*parts)
    return np.stack(mu), np.stack(us)


def subspace_head_scores(q: np.ndarray, mu: np.ndarray, us: np.ndarray, p: np.ndarray,
                         n_tokens: np.ndarray) -> np.ndarray:
    """s_b = ln n_b + (q.mu_b)/sqrt(d) + 1/2 |U_s,b^T (P^T q)|^2 / d."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[0]
    qs = np.asarray(p, dtype=np.float64).T @ q              # query in subspace coordinates
    linear = mu @ q / math.sqrt(d)
    proj = us @ qs                                         # [nb, r]
    quadratic = 0.5 * np.sum(proj * proj, axis=1) / d
    return np.log(np.asarray(n_tokens, dtype=np.float64)) + linear + quadratic


def subspace_group_scores(q_group, mu, us, p, n_tokens) -> np.ndarray:
    """S_b = ln sum_h exp(s_{h,b}) over the G query heads of one kv-head."""
    per_head = np.stack([subspace_head_scores(q, mu, us, p, n_tokens)
                         for q in np.asarray(q_group, dtype=np.float64)], axis=0)
    return _logsumexp(per_head, axis=0)


def select_from_subspace_records(q_group, mu, us, p, seq_len, block, top_k, sink_blocks,
                                 local_tokens):
    """Score every complete block from its subspace record, then select."""
    n_full = seq_len // block
    scores = subspace_group_scores(q_group, mu[:n_full], us[:n_full], p,
                                   np.full(n_full, block))
    return select_blocks(scores, seq_len, block, top_k, sink_blocks,
                         local_tokens), scores
