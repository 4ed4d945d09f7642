"""Helpers shared by the GPU parity tests (test infrastructure).

Moves seeded inputs from ``workloads`` onto the device, calls the three C-ABI
entry points through the Python binding, and compares against the oracle
with the tolerances the tests use:

* attention outputs: max-abs error 2e-3 (bf16 inputs, fp32 accumulation);
  lse: 1e-3;
* selected blocks: identical, except where two blocks' oracle fp64 scores at
  the top-k boundary differ by at most 1e-5 * max(1, |S|) (a reported tie);
* block statistics: mu within one bf16 step of the oracle's rounded fp64
  mean; projector U U^T within 1e-2 relative Frobenius error on blocks whose
  oracle spectrum has lambda_r / lambda_{r+1} >= 1.05; captured energy
  trace(U U^T) >= (1 - 1e-3) of the oracle's on every block.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from workloads import bits_to_f64, make_kv, make_queries

OUT_ATOL = 2e-3
LSE_ATOL = 1e-3
TIE_RTOL = 1e-5
PROJ_RTOL = 1e-2
GAP_MIN = 1.05
ENERGY_RTOL = 1e-3


def dims_of(w, **kw):
    d = dict(batch=w.batch, num_q_heads=w.q_heads, num_kv_heads=w.kv_heads,
             head_dim=w.head_dim, block_size=w.block, rank=w.rank,
             capacity_tokens=w.cap)
    d.update(kw)
    return d


def to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda()


def from_dev_bits(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


class Problem:
    """Device buffers for one workload (inputs, stats, selection, outputs)."""

    def __init__(self, w, poison="zero", workers=1, q_step=0):
        self.w = w
        self.q_bits = make_queries(w, q_step)
        self.k_bits, self.v_bits = make_kv(w, make_queries(w, 0) if w.needles else None,
                                           poison=poison, workers=workers)
        self.dims = dims_of(w)
        self.q = to_dev(self.q_bits)
        self.k = to_dev(self.k_bits)
        self.v = to_dev(self.v_bits)
        nb_cap = w.cap // w.block
        self.stats = torch.zeros((w.batch, w.kv_heads, nb_cap, 1 + w.rank, w.head_dim),
                                 dtype=torch.int16, device="cuda")
        self.nsm = cb.cobs_selected_capacity(self.dims, w.top_k, w.sink_blocks,
                                             w.local_tokens)
        self.idx = torch.full((w.batch, w.kv_heads, self.nsm), -7, dtype=torch.int32,
                              device="cuda")
        self.n_sel = torch.zeros((w.batch, w.kv_heads), dtype=torch.int32, device="cuda")
        self.scores = torch.full((w.batch, w.kv_heads, nb_cap), float("nan"),
                                 dtype=torch.float32, device="cuda")
        self.out = torch.zeros((w.batch, w.q_heads, w.head_dim), dtype=torch.float32,
                               device="cuda")
        self.lse = torch.zeros((w.batch, w.q_heads), dtype=torch.float32, device="cuda")
        self.ws_bytes = cb.cobs_workspace_bytes(self.dims, w.top_k, w.sink_blocks,
                                                w.local_tokens)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        cb.cobs_workspace_init(self.ws, self.ws_bytes)

    # ---- the three calls ------------------------------------------------------
    def build_stats(self, begin=0, end=None):
        end = self.w.seq_len // self.w.block if end is None else end
        cb.cobs_build_block_stats(self.dims, self.k, begin, end, self.stats, self.ws,
                                  self.ws_bytes)

    def select(self, seq_len=None, top_k=None, sink=None, local=None, scores=True):
        w = self.w
        cb.cobs_select_blocks(self.dims, self.q, self.stats,
                              w.seq_len if seq_len is None else seq_len,
                              w.top_k if top_k is None else top_k,
                              w.sink_blocks if sink is None else sink,
                              w.local_tokens if local is None else local,
                              self.idx, self.idx.shape[-1], self.n_sel,
                              self.scores if scores else None,
                              self.ws, self.ws_bytes)

    def decode(self, seq_len=None, idx=None, n_sel=None, stride=None):
        w = self.w
        idx = self.idx if idx is None else idx
        n_sel = self.n_sel if n_sel is None else n_sel
        cb.cobs_sparse_decode(self.dims, self.q, self.k, self.v, idx, n_sel,
                              idx.shape[-1] if stride is None else stride,
                              w.seq_len if seq_len is None else seq_len,
                              1.0 / math.sqrt(w.head_dim), self.out, self.lse, self.ws,
                              self.ws_bytes)

    def device_status(self):
        return cb.cobs_read_device_status(self.ws, self.ws_bytes)

    # ---- oracle-side views ----------------------------------------------------
    def q_group(self, b, h):
        G = self.w.group
        return bits_to_f64(self.q_bits[b, h * G:(h + 1) * G])

    def keys(self, b, h):
        return bits_to_f64(self.k_bits[b, h])

    def values(self, b, h):
        return bits_to_f64(self.v_bits[b, h])

    def oracle_records(self, b, h, n_blocks=None):
        w = self.w
        n = w.seq_len // w.block if n_blocks is None else n_blocks
        return O.build_block_records(self.keys(b, h), w.block, w.rank, 0, n)

    def upload_records(self, b, h, recs):
        bits = _f64_to_bf16_bits(recs)
        self.stats[b, h, :recs.shape[0]] = to_dev(bits)


def _f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Exact bf16 values (fp64) -> their bit patterns."""
    f32 = np.ascontiguousarray(x, dtype=np.float32)
    u = f32.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "values are not bf16-representable"
    return (u >> 16).astype(np.uint16)


def selection_mismatch(gpu_sel, orc_sel, orc_scores, w, seq_len=None):
    """Blocks that differ between the selections and are not score ties.

    Returns a list of (block, oracle score, boundary score) for offending
    blocks; empty when the selections agree up to reported ties."""
    seq_len = w.seq_len if seq_len is None else seq_len
    a, b = set(int(x) for x in gpu_sel), set(int(x) for x in orc_sel)
    diff = a ^ b
    if not diff:
        return []
    forced, c0, c1 = O.block_partition(seq_len, w.block, w.sink_blocks, w.local_tokens)
    cand = np.arange(c0, c1)
    s = np.asarray(orc_scores)[c0:c1]
    order = np.lexsort((cand, -s))
    k = min(w.top_k, len(cand))
    boundary = s[order[k - 1]] if k > 0 else -np.inf
    bad = []
    for j in sorted(diff):
        if j in forced or not (c0 <= j < c1):
            bad.append((j, float("nan"), float(boundary)))
            continue
        sj = orc_scores[j]
        if abs(sj - boundary) > TIE_RTOL * max(1.0, abs(boundary)):
            bad.append((j, float(sj), float(boundary)))
    return bad


def stats_errors(gpu_rec, orc_rec, orc_keys_block, rank):
    """(mu ok, projector rel error or None if not gapped, energy ratio)."""
    mu_g, mu_o = gpu_rec[0], orc_rec[0]
    # one bf16 step of the oracle's mean, with an absolute floor for means
    # near zero (fp32 summation error of 64 keys)
    floor = 1e-6 * max(1.0, float(np.max(np.abs(orc_keys_block))))
    step = np.maximum(np.abs(mu_o) * 2.0 ** -7, floor)
    mu_ok = bool(np.all(np.abs(mu_g - mu_o) <= step * 1.0001))
    if rank == 0:
        return mu_ok, 0.0, 1.0
    ug, uo = gpu_rec[1:].T, orc_rec[1:].T
    pg, po = ug @ ug.T, uo @ uo.T
    _, sigma = O.block_moments(orc_keys_block)
    lam = np.sort(np.linalg.eigvalsh(sigma))[::-1]
    gapped = lam[rank] <= 0 or lam[rank - 1] / lam[rank] >= GAP_MIN
    rel = float(np.linalg.norm(pg - po) / max(np.linalg.norm(po), 1e-30)) if gapped else None
    tr_o = float(np.trace(po))
    energy = float(np.trace(pg) / tr_o) if tr_o > 0 else 1.0
    return mu_ok, rel, energy


# ---- FP4 records: the byte layout of include/cobs.h (cobs_dims.stats_format) ----

def fp4_record_bytes(d, r):
    return (2 * d + r * (d // 2) + r * (d // 32) + 15) // 16 * 16


def pack_fp4_records(mu, codes, scale_bytes):
    """Oracle FP4 records (mu [nb, d] exact bf16 values, codes [nb, r, d],
    scale bytes [nb, r, d/32]) -> [nb, record bytes] uint8."""
    nb, r, d = codes.shape
    out = np.zeros((nb, fp4_record_bytes(d, r)), dtype=np.uint8)
    out[:, :2 * d] = _f64_to_bf16_bits(mu).reshape(nb, d).view(np.uint8).reshape(nb, 2 * d)
    packed = (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)
    c0 = 2 * d
    out[:, c0:c0 + r * d // 2] = packed.reshape(nb, -1)
    s0 = c0 + r * d // 2
    out[:, s0:s0 + r * d // 32] = scale_bytes.reshape(nb, -1)
    return out


def unpack_fp4_records(raw, d, r):
    """[nb, record bytes] uint8 -> (mu as fp64, codes, scale bytes, padding bytes)."""
    raw = np.ascontiguousarray(raw, dtype=np.uint8)
    nb = raw.shape[0]
    mu = bits_to_f64(raw[:, :2 * d].copy().view(np.uint16))
    c0 = 2 * d
    packed = raw[:, c0:c0 + r * d // 2].reshape(nb, r, d // 2)
    codes = np.empty((nb, r, d), dtype=np.uint8)
    codes[..., 0::2] = packed & 15
    codes[..., 1::2] = packed >> 4
    s0 = c0 + r * d // 2
    sb = raw[:, s0:s0 + r * d // 32].reshape(nb, r, d // 32)
    return mu, codes, sb, raw[:, s0 + r * d // 32:]


class Fp4Problem(Problem):
    """A Problem whose block records are FP4 (COBS_STATS_FP4)."""

    def __init__(self, w, **kw):
        super().__init__(w, **kw)
        self.dims4 = dict(self.dims, stats_format=cb.COBS_STATS_FP4)
        self.rec = cb.cobs_stats_record_bytes(self.dims4)
        assert self.rec == fp4_record_bytes(w.head_dim, w.rank)
        self.stats4 = torch.zeros((w.batch, w.kv_heads, w.cap // w.block, self.rec),
                                  dtype=torch.uint8, device="cuda")

    def build_stats4(self, begin=0, end=None):
        end = self.w.seq_len // self.w.block if end is None else end
        cb.cobs_build_block_stats(self.dims4, self.k, begin, end, self.stats4, self.ws,
                                  self.ws_bytes)

    def select4(self, seq_len=None):
        w = self.w
        cb.cobs_select_blocks(self.dims4, self.q, self.stats4,
                              w.seq_len if seq_len is None else seq_len, w.top_k,
                              w.sink_blocks, w.local_tokens, self.idx, self.idx.shape[-1],
                              self.n_sel, self.scores, self.ws, self.ws_bytes)

    def oracle_records4(self, b, h, n_blocks=None):
        w = self.w
        n = w.seq_len // w.block if n_blocks is None else n_blocks
        return O.build_block_records_fp4(self.keys(b, h), w.block, w.rank, 0, n)

    def upload_records4(self, b, h, parts):
        raw = pack_fp4_records(*parts)
        self.stats4[b, h, :raw.shape[0]] = torch.from_numpy(raw).cuda()


def explain_selection(w, q_group, gpu_sel, gpu_recs, orc_recs, seq_len=None):
    """End-to-end selection check that explains every flip.

    ``gpu_recs`` are the records the GPU built (as fp64 values), ``orc_recs``
    the oracle's, both [n_full, 1 + r, d].  Two facts are asserted:

    1. The GPU selection is the oracle's selection rule applied to the GPU's
       own records (up to reported ties): the selection kernel adds nothing.
    2. Every block in which the GPU and the oracle selections differ has an
       oracle score within 2 Delta (+ the tie tolerance) of the oracle's top-k
       boundary, Delta = max over candidates |S(gpu record) - S(oracle record)|.
       Moving every score by at most Delta moves the k-th largest by at most
       Delta, so a block can only cross the boundary from within 2 Delta.

    Returns (number of differing blocks, Delta, list of (block, oracle score,
    boundary, per-block score change) for the differing blocks)."""
    seq_len = w.seq_len if seq_len is None else seq_len
    n_full = seq_len // w.block
    n_tok = np.full(n_full, w.block)
    s_g = O.group_block_scores(q_group, gpu_recs[:n_full], n_tok)
    s_o = O.group_block_scores(q_group, orc_recs[:n_full], n_tok)
    sel_g = O.select_blocks(s_g, seq_len, w.block, w.top_k, w.sink_blocks, w.local_tokens)
    assert selection_mismatch(gpu_sel, sel_g, s_g, w, seq_len) == [], "selection vs own records"
    sel_o = O.select_blocks(s_o, seq_len, w.block, w.top_k, w.sink_blocks, w.local_tokens)
    _, c0, c1 = O.block_partition(seq_len, w.block, w.sink_blocks, w.local_tokens)
    if c1 <= c0:
        assert set(int(x) for x in gpu_sel) == set(int(x) for x in sel_o)
        return 0, 0.0, []
    delta = float(np.max(np.abs(s_g[c0:c1] - s_o[c0:c1])))
    cand = np.arange(c0, c1)
    order = np.lexsort((cand, -s_o[c0:c1]))
    k = min(w.top_k, c1 - c0)
    boundary = float(s_o[c0:c1][order[k - 1]]) if k > 0 else -np.inf
    diff = sorted(set(int(x) for x in gpu_sel) ^ set(int(x) for x in sel_o))
    rows = []
    for j in diff:
        assert c0 <= j < c1, ("forced block differs", j)
        slack = 2 * delta + TIE_RTOL * max(1.0, abs(boundary))
        assert abs(s_o[j] - boundary) <= slack, (j, float(s_o[j]), boundary, delta)
        rows.append((j, float(s_o[j]), boundary, float(abs(s_g[j] - s_o[j]))))
    return len(diff), delta, rows


def score_change_bound(q_group, orc_rec, rank):
    """A-priori bound of |s_h(GPU record) - s_h(oracle record)| over the heads
    of one block when the GPU record meets the statistics tolerance: each mean
    component within one bf16 step (|d mu| <= 2^-7 |mu|) and the projector
    within PROJ_RTOL (relative Frobenius) of the oracle's:
        |q.d mu| / sqrt(d) + 1/2 |q|^2 |d Sigma_r|_2 / d
        <= |q| 2^-7 |mu| / sqrt(d) + 1/2 |q|^2 PROJ_RTOL |Sigma_r|_F / d."""
    d = orc_rec.shape[1]
    mu, u = orc_rec[0], orc_rec[1:1 + rank].T
    proj_f = float(np.linalg.norm(u @ u.T)) if rank else 0.0
    qn = np.linalg.norm(np.asarray(q_group, dtype=np.float64), axis=1)
    return float(np.max(qn * 2.0 ** -7 * np.linalg.norm(mu) / math.sqrt(d)
                        + 0.5 * qn ** 2 * PROJ_RTOL * proj_f / d))


def block_is_gapped(keys_block, rank):
    """Whether the block's covariance spectrum fixes its top-r subspace
    (lambda_r / lambda_{r+1} >= GAP_MIN, or lambda_{r+1} = 0)."""
    if rank == 0:
        return True
    _, sigma = O.block_moments(keys_block)
    lam = np.sort(np.linalg.eigvalsh(sigma))[::-1]
    return bool(lam[rank] <= 0 or lam[rank - 1] / lam[rank] >= GAP_MIN)
