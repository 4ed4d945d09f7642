"""Subspace records (COBS explainer §2.3, subspace projection; §4.3: an
adaptive s of about 85 of 128 matches the full dimension) on the GPU against
the oracle.

Reading taken (the pages give no formula beyond "the covariance projected on
the query subspace"): the basis P is the top-s eigenvectors of the queries'
uncentred second moment M = (1/n) sum q q^T over calibration queries; a block
stores mu in full and U_s = P^T U; the score's quadratic term is
1/2 |U_s^T P^T q|^2 / d.  Calibration queries here are seeded draws with a
planted anisotropy (there is no trained model); P is rounded to fp32, the
precision the library takes it in, and the oracle uses the same rounded P.

* Statistics: mu as in the bf16 build; U_s U_s^T within the projector
  tolerance of the oracle's P^T Sigma_r P on blocks whose spectrum fixes the
  top-r subspace; padding columns zero.
* Selection over oracle subspace records: the oracle's selection up to
  reported ties, scores within the tie tolerance; also at the full 32k
  batched size.
* End to end: every selection flip explained by the records, outputs equal
  to the oracle's attention over the GPU's selection.
* s = d with P = I: the same scores as bf16 COBS records of the same factor.
"""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from harness import (GAP_MIN, OUT_ATOL, PROJ_RTOL, TIE_RTOL, Problem, _f64_to_bf16_bits,
                     block_is_gapped, from_dev_bits, selection_mismatch, to_dev)
from workloads import WORKLOADS, bits_to_f64, make_kv_slice, make_queries

pytestmark = pytest.mark.gpu

W = WORKLOADS
CASES = {
    "needles_b2_s85": (W["batched_needles_32k"].scaled(batch=2, seq_len=4096 + 37), 85),
    "g8_r16_s96": (W["build_256k"].scaled(seq_len=8192, append_chunk=0, decode_steps=1), 96),
    "g1_r8_s64": (W["single_32k"].scaled(q_heads=2, kv_heads=2, seq_len=3000, top_k=5,
                                         local_tokens=100), 64),
    "g2_r4_s17_many": (W["single_32k"].scaled(q_heads=4, kv_heads=2, rank=4, seq_len=80000,
                                              top_k=200, local_tokens=0), 17),
    "d64_g8_r8_s40": (W["tiny_4k"].scaled(q_heads=8, kv_heads=1, rank=8, seq_len=2500,
                                          batch=3), 40),
    "d64_g4_r4_s64": (W["tiny_4k"], 64),
}


def pad8(s):
    return (s + 7) // 8 * 8


def calibration_basis(w, s, seed=5):
    """Per kv-head basis [Hkv, s, d] (fp32 values as fp64) from seeded
    calibration queries with a planted anisotropy."""
    rng = np.random.default_rng(seed)
    d = w.head_dim
    out = np.zeros((w.kv_heads, s, d))
    for h in range(w.kv_heads):
        a = rng.standard_normal((d, d)) * np.exp(-np.arange(d) / (0.4 * d))[None, :]
        q_cal = rng.standard_normal((4096, d)) @ a.T + 0.2 * rng.standard_normal(d)
        p = O.query_subspace(q_cal, s)                          # [d, s]
        out[h] = p.T.astype(np.float32).astype(np.float64)
    return out


def pack_subspace_records(mu, us, s8):
    """(mu [nb, d] exact bf16 values, us [nb, r, s]) -> [nb, bytes] uint8."""
    nb, r, s = us.shape
    d = mu.shape[1]
    rows = np.zeros((nb, r, s8))
    rows[:, :, :s] = us
    out = np.zeros((nb, 2 * d + 2 * r * s8), dtype=np.uint8)
    out[:, :2 * d] = _f64_to_bf16_bits(mu).view(np.uint8).reshape(nb, 2 * d)
    out[:, 2 * d:] = _f64_to_bf16_bits(rows).reshape(nb, r * s8).view(np.uint8)
    return out


def unpack_subspace_records(raw, d, r, s):
    s8 = pad8(s)
    raw = np.ascontiguousarray(raw)
    nb = raw.shape[0]
    mu = bits_to_f64(raw[:, :2 * d].copy().view(np.uint16))
    rows = bits_to_f64(raw[:, 2 * d:2 * d + 2 * r * s8].copy().view(np.uint16)).reshape(nb, r, s8)
    return mu, rows[:, :, :s], rows[:, :, s:]


class SubProblem(Problem):
    def __init__(self, w, s, **kw):
        super().__init__(w, **kw)
        self.s = s
        self.P = calibration_basis(w, s)                       # [Hkv, s, d]
        self.basis = torch.from_numpy(self.P.astype(np.float32)).cuda()
        self.dimss = dict(self.dims, stats_format=cb.COBS_STATS_SUBSPACE, subspace_dim=s,
                          subspace_basis=self.basis)
        self.rec = cb.cobs_stats_record_bytes(self.dimss)
        assert self.rec == 2 * w.head_dim + 2 * w.rank * pad8(s)
        self.stats_s = torch.zeros((w.batch, w.kv_heads, w.cap // w.block, self.rec),
                                   dtype=torch.uint8, device="cuda")

    def p_of(self, h):
        return self.P[h].T                                      # [d, s] as the oracle takes it

    def build_sub(self, begin=0, end=None):
        end = self.w.seq_len // self.w.block if end is None else end
        cb.cobs_build_block_stats(self.dimss, self.k, begin, end, self.stats_s, self.ws,
                                  self.ws_bytes)

    def select_sub(self):
        w = self.w
        cb.cobs_select_blocks(self.dimss, self.q, self.stats_s, w.seq_len, w.top_k,
                              w.sink_blocks, w.local_tokens, self.idx, self.idx.shape[-1],
                              self.n_sel, self.scores, self.ws, self.ws_bytes)

    def oracle_sub(self, b, h):
        w = self.w
        return O.build_block_records_subspace(self.keys(b, h), w.block, w.rank, self.p_of(h), 0,
                                              w.seq_len // w.block)


@pytest.fixture(scope="module", params=list(CASES))
def sp(request):
    torch.cuda.synchronize()
    w, s = CASES[request.param]
    return SubProblem(w, s, poison="nan")


def test_subspace_stats(sp):
    p, w = sp, sp.w
    d, r, s = w.head_dim, w.rank, sp.s
    nfull = w.seq_len // w.block
    p.build_sub()
    raw = p.stats_s.cpu().numpy()
    rng = np.random.default_rng(2)
    checked = 0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            keys = p.keys(b, h)
            mu_g, us_g, pad = unpack_subspace_records(raw[b, h, :nfull], d, r, s)
            assert np.all(pad == 0)
            ph = p.p_of(h)
            for j in sorted(set(rng.choice(nfull, size=min(nfull, 40), replace=False))):
                kb = keys[j * 64:(j + 1) * 64]
                mu_o, sigma = O.block_moments(kb)
                step = np.maximum(np.abs(O.round_to_bf16(mu_o)) * 2.0 ** -7, 1e-6)
                assert np.all(np.abs(mu_g[j] - mu_o) <= step * 1.0001), (b, h, j)
                if not block_is_gapped(kb, r):
                    continue
                u_o, _ = O.covariance_factor(sigma, r)
                po = ph.T @ (u_o @ u_o.T) @ ph                  # P^T Sigma_r P
                pg = us_g[j].T @ us_g[j]
                rel = np.linalg.norm(pg - po) / max(np.linalg.norm(po), 1e-30)
                assert rel <= PROJ_RTOL, (b, h, j, rel)
                checked += 1
    assert checked > 0
    assert p.device_status() == 0


def test_subspace_select_on_oracle_records(sp):
    p, w = sp, sp.w
    nfull = w.seq_len // w.block
    s8 = pad8(sp.s)
    orc = {}
    for b in range(w.batch):
        for h in range(w.kv_heads):
            mu, us = p.oracle_sub(b, h)
            p.stats_s[b, h, :nfull] = torch.from_numpy(pack_subspace_records(mu, us, s8)).cuda()
            orc[(b, h)] = O.select_from_subspace_records(p.q_group(b, h), mu, us, p.p_of(h),
                                                         w.seq_len, w.block, w.top_k,
                                                         w.sink_blocks, w.local_tokens)
    p.select_sub()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    scores = p.scores.cpu().numpy()
    _, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
    for (b, h), (sel, sc) in orc.items():
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0) and n[b, h] == len(sel)
        assert selection_mismatch(got, sel, sc, w) == [], (b, h)
        if c1 > c0:
            np.testing.assert_allclose(scores[b, h, c0:c1], sc[c0:c1], rtol=0,
                                       atol=TIE_RTOL * max(1, np.max(np.abs(sc))))
    assert p.device_status() == 0


def test_subspace_end_to_end(sp):
    p, w = sp, sp.w
    d, r, s = w.head_dim, w.rank, sp.s
    nfull = w.seq_len // w.block
    p.build_sub()
    p.select_sub()
    p.decode()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    out = p.out.cpu().numpy()
    raw = p.stats_s.cpu().numpy()
    G = w.group
    scale = 1 / math.sqrt(d)
    n_tok = np.full(nfull, w.block)
    flips = 0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            qg = p.q_group(b, h)
            mu_g, us_g, _ = unpack_subspace_records(raw[b, h, :nfull], d, r, s)
            mu_o, us_o = p.oracle_sub(b, h)
            ph = p.p_of(h)
            s_g = O.subspace_group_scores(qg, mu_g, us_g, ph, n_tok)
            s_o = O.subspace_group_scores(qg, mu_o, us_o, ph, n_tok)
            got = idx[b, h, :n[b, h]]
            sel_g = O.select_blocks(s_g, w.seq_len, w.block, w.top_k, w.sink_blocks,
                                    w.local_tokens)
            assert selection_mismatch(got, sel_g, s_g, w) == [], (b, h)   # its own records
            sel_o = O.select_blocks(s_o, w.seq_len, w.block, w.top_k, w.sink_blocks,
                                    w.local_tokens)
            _, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
            diff = set(got.tolist()) ^ set(sel_o.tolist())
            if diff and c1 > c0:
                flips += 1
                delta = float(np.max(np.abs(s_g[c0:c1] - s_o[c0:c1])))
                cand = np.arange(c0, c1)
                order = np.lexsort((cand, -s_o[c0:c1]))
                bound = s_o[c0:c1][order[min(w.top_k, c1 - c0) - 1]]
                for j in diff:
                    assert abs(s_o[j] - bound) <= 2 * delta + TIE_RTOL * max(1, abs(bound))
            o, _ = O.sparse_attention(qg, p.keys(b, h), p.values(b, h), got.astype(np.int64),
                                      w.seq_len, w.block, scale)
            assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL
    print(f"subspace end-to-end selections differing from the oracle's: {flips} of "
          f"{w.batch * w.kv_heads} (each explained by its records)")
    assert p.device_status() == 0


def test_full_subspace_equals_bf16_records():
    """s = d with P = I: U_s = U, so the subspace records hold the bf16
    records' numbers and the selection gives the same scores."""
    w = W["single_32k"].scaled(batch=2, seq_len=4096 + 64 * 5)
    p = Problem(w)
    d = w.head_dim
    eye = torch.eye(d, dtype=torch.float32, device="cuda").repeat(w.kv_heads, 1, 1).contiguous()
    dims = dict(p.dims, stats_format=cb.COBS_STATS_SUBSPACE, subspace_dim=d, subspace_basis=eye)
    rec = cb.cobs_stats_record_bytes(dims)
    assert rec == (1 + w.rank) * d * 2
    st = torch.zeros((w.batch, w.kv_heads, w.cap // w.block, rec), dtype=torch.uint8,
                     device="cuda")
    nfull = w.seq_len // w.block
    p.build_stats()
    cb.cobs_build_block_stats(dims, p.k, 0, nfull, st, p.ws, p.ws_bytes)
    torch.cuda.synchronize()
    bf = p.stats.view(torch.uint8).reshape(st.shape)
    assert torch.equal(st[:, :, :nfull], bf[:, :, :nfull])
    p.select()
    want_idx, want_n, want_s = p.idx.clone(), p.n_sel.clone(), p.scores.clone()
    p.scores.fill_(float("nan"))
    cb.cobs_select_blocks(dims, p.q, st, w.seq_len, w.top_k, w.sink_blocks, w.local_tokens,
                          p.idx, p.idx.shape[-1], p.n_sel, p.scores, p.ws, p.ws_bytes)
    torch.cuda.synchronize()
    assert torch.equal(p.n_sel, want_n)
    _, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
    ds = (p.scores[:, :, c0:c1] - want_s[:, :, c0:c1]).abs().max().item()
    assert ds <= TIE_RTOL * max(1.0, want_s[:, :, c0:c1].abs().max().item())
    assert p.device_status() == 0


def test_subspace_select_at_full_size():
    """Subspace selection in the launch the full 32k batched workload gets,
    on sampled pairs with the oracle's records uploaded (s = 85)."""
    w, s = W["batched_needles_32k"], 85
    q_bits = make_queries(w)
    P = calibration_basis(w, s)
    basis = torch.from_numpy(P.astype(np.float32)).cuda()
    dims = dict(batch=w.batch, num_q_heads=w.q_heads, num_kv_heads=w.kv_heads,
                head_dim=w.head_dim, block_size=w.block, rank=w.rank, capacity_tokens=w.cap,
                stats_format=cb.COBS_STATS_SUBSPACE, subspace_dim=s, subspace_basis=basis)
    rec = cb.cobs_stats_record_bytes(dims)
    nb_cap, nfull = w.cap // w.block, w.seq_len // w.block
    st = torch.zeros((w.batch, w.kv_heads, nb_cap, rec), dtype=torch.uint8, device="cuda")
    q = to_dev(q_bits)
    nsm = cb.cobs_selected_capacity(dims, w.top_k, w.sink_blocks, w.local_tokens)
    idx = torch.zeros((w.batch, w.kv_heads, nsm), dtype=torch.int32, device="cuda")
    n_sel = torch.zeros((w.batch, w.kv_heads), dtype=torch.int32, device="cuda")
    ws_bytes = cb.cobs_workspace_bytes(dims, w.top_k, w.sink_blocks, w.local_tokens)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    cb.cobs_workspace_init(ws, ws_bytes)
    G = w.group
    orc = {}
    for (b, h) in [(0, 0), (21, 3), (31, 7)]:
        kb, _ = make_kv_slice(w, b, h, q_bits)
        mu, us = O.build_block_records_subspace(bits_to_f64(kb), w.block, w.rank, P[h].T, 0,
                                                nfull)
        st[b, h, :nfull] = torch.from_numpy(pack_subspace_records(mu, us, pad8(s))).cuda()
        orc[(b, h)] = O.select_from_subspace_records(bits_to_f64(q_bits[b, h * G:(h + 1) * G]),
                                                     mu, us, P[h].T, w.seq_len, w.block,
                                                     w.top_k, w.sink_blocks, w.local_tokens)
    cb.cobs_select_blocks(dims, q, st, w.seq_len, w.top_k, w.sink_blocks, w.local_tokens, idx,
                          nsm, n_sel, None, ws, ws_bytes)
    idx_h, n_h = idx.cpu().numpy(), n_sel.cpu().numpy()
    for (b, h), (sel, sc) in orc.items():
        got = idx_h[b, h, :n_h[b, h]]
        assert len(got) == len(sel) and selection_mismatch(got, sel, sc, w) == [], (b, h)
    assert cb.cobs_read_device_status(ws, ws_bytes) == 0
