"""Per-sequence lengths (ragged batches) on the GPU against the oracle.

Every sequence has its own block partition (sink blocks, its own local window
and tail block, the complete blocks between as candidates).  Tokens past a
sequence are NaN in the cache, and the records of blocks past it are NaN in
the statistics, so any read of them shows up in the results."""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from harness import LSE_ATOL, OUT_ATOL, Problem, selection_mismatch
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu

W = WORKLOADS
NAN_BITS = 0x7FC0
CASES = {
    "d128_g4": (W["single_32k"].scaled(batch=4, q_heads=8, kv_heads=2, seq_len=4096 + 37),
                [4096 + 37, 3500 + 3, 1000 + 1, 130]),
    "d128_g8_r16": (W["build_256k"].scaled(batch=3, seq_len=8192 + 5, append_chunk=0,
                                           decode_steps=1),
                    [8192 + 5, 6000, 2500 + 63]),
    "d64_g8": (W["tiny_4k"].scaled(batch=3, q_heads=8, kv_heads=1, rank=8, seq_len=2500),
               [2500, 1777, 64]),
}


class Ragged:
    def __init__(self, w, lens):
        self.p = Problem(w)
        self.w, self.lens = w, lens
        self.seq_lens = torch.tensor(lens, dtype=torch.int64, device="cuda")
        p = self.p
        for b, L in enumerate(lens):
            p.k[b, :, L:w.seq_len] = NAN_BITS
            p.v[b, :, L:w.seq_len] = NAN_BITS
        self.recs = {}
        for b, L in enumerate(lens):
            for h in range(w.kv_heads):
                r = O.build_block_records(p.keys(b, h)[:L], w.block, w.rank, 0, L // w.block)
                self.recs[(b, h)] = r

    def upload_oracle_stats(self):
        p, w = self.p, self.w
        p.stats.fill_(NAN_BITS)
        for (b, h), r in self.recs.items():
            if r.shape[0]:
                p.upload_records(b, h, r)

    def select(self):
        p, w = self.p, self.w
        cb.cobs_select_blocks_varlen(p.dims, p.q, p.stats, self.seq_lens, w.seq_len, w.top_k,
                                     w.sink_blocks, w.local_tokens, p.idx, p.idx.shape[-1],
                                     p.n_sel, None, p.ws, p.ws_bytes)

    def decode(self, idx, n):
        p, w = self.p, self.w
        cb.cobs_sparse_decode_varlen(p.dims, p.q, p.k, p.v, idx, n, idx.shape[-1],
                                     self.seq_lens, w.seq_len, 1.0 / math.sqrt(w.head_dim),
                                     p.out, p.lse, p.ws, p.ws_bytes)

    def oracle_selection(self, b, h):
        w = self.w
        return O.select_from_records(self.p.q_group(b, h), self.recs[(b, h)], self.lens[b],
                                     w.block, w.top_k, w.sink_blocks, w.local_tokens)


@pytest.fixture(scope="module", params=list(CASES))
def rag(request):
    w, lens = CASES[request.param]
    return Ragged(w, lens)


def test_varlen_select_on_oracle_stats(rag):
    rag.upload_oracle_stats()
    rag.select()
    idx, n = rag.p.idx.cpu().numpy(), rag.p.n_sel.cpu().numpy()
    w = rag.w
    for (b, h) in rag.recs:
        sel, s = rag.oracle_selection(b, h)
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0), (b, h)
        assert len(got) == len(sel), (b, h)
        assert selection_mismatch(got, sel, s, w, rag.lens[b]) == [], (b, h)
    assert rag.p.device_status() == 0


def test_varlen_decode_on_oracle_selection(rag):
    p, w = rag.p, rag.w
    idx = torch.zeros_like(p.idx)
    n = torch.zeros_like(p.n_sel)
    sels = {}
    for (b, h) in rag.recs:
        sel, _ = rag.oracle_selection(b, h)
        sels[(b, h)] = sel
        idx[b, h, :len(sel)] = torch.tensor(sel.astype(np.int32), device="cuda")
        n[b, h] = len(sel)
    rag.decode(idx, n)
    out, lse = p.out.cpu().numpy(), p.lse.cpu().numpy()
    G = w.group
    scale = 1.0 / math.sqrt(w.head_dim)
    for (b, h), sel in sels.items():
        L = rag.lens[b]
        o, l = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h), sel, L,
                                  w.block, scale)
        assert np.all(np.isfinite(out[b, h * G:(h + 1) * G]))
        assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL, (b, h)
        np.testing.assert_allclose(lse[b, h * G:(h + 1) * G], l, atol=LSE_ATOL)
    assert p.device_status() == 0


def test_varlen_end_to_end_per_sequence_stats(rag):
    """Each sequence's complete blocks built on the GPU (a batch-1 call on its
    slice), then ragged selection and decode; flips on near-degenerate spectra
    are reported, outputs compared wherever the selections agree."""
    p, w = rag.p, rag.w
    p.stats.fill_(NAN_BITS)
    d1 = dict(p.dims, batch=1)
    for b, L in enumerate(rag.lens):
        if L // w.block:
            cb.cobs_build_block_stats(d1, p.k[b], 0, L // w.block, p.stats[b], p.ws, p.ws_bytes)
    rag.select()
    rag.decode(p.idx, p.n_sel)
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    out = p.out.cpu().numpy()
    G = w.group
    flips = 0
    for (b, h) in rag.recs:
        sel, _ = rag.oracle_selection(b, h)
        got = idx[b, h, :n[b, h]]
        assert len(got) == len(sel)
        assert np.all(np.isfinite(out[b, h * G:(h + 1) * G]))
        if set(got.tolist()) != set(sel.tolist()):
            flips += 1
            continue
        o, _ = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h), sel,
                                  rag.lens[b], w.block, 1.0 / math.sqrt(w.head_dim))
        assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL
    print(f"ragged end-to-end: selection flips on {flips} of {len(rag.recs)} pairs")
    assert p.device_status() == 0


def test_varlen_with_equal_lengths_matches_the_single_length_calls():
    w = W["single_32k"].scaled(batch=2, q_heads=8, kv_heads=2, seq_len=3000 + 11)
    p = Problem(w)
    p.build_stats()
    p.select()
    p.decode()
    torch.cuda.synchronize()
    idx1, n1, out1, lse1 = p.idx.clone(), p.n_sel.clone(), p.out.clone(), p.lse.clone()
    lens = torch.full((w.batch,), w.seq_len, dtype=torch.int64, device="cuda")
    p.idx.fill_(-5)
    cb.cobs_select_blocks_varlen(p.dims, p.q, p.stats, lens, w.seq_len, w.top_k,
                                 w.sink_blocks, w.local_tokens, p.idx, p.idx.shape[-1],
                                 p.n_sel, None, p.ws, p.ws_bytes)
    cb.cobs_sparse_decode_varlen(p.dims, p.q, p.k, p.v, p.idx, p.n_sel, p.idx.shape[-1], lens,
                                 w.seq_len, 1.0 / math.sqrt(w.head_dim), p.out, p.lse, p.ws,
                                 p.ws_bytes)
    torch.cuda.synchronize()
    assert torch.equal(p.n_sel, n1)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            assert torch.equal(p.idx[b, h, :n1[b, h]], idx1[b, h, :n1[b, h]])
    assert torch.equal(p.out, out1) and torch.equal(p.lse, lse1)
    assert p.device_status() == 0


def test_varlen_out_of_range_length_is_reported():
    w = W["single_32k"].scaled(batch=2, q_heads=8, kv_heads=2, seq_len=2048)
    p = Problem(w)
    p.build_stats()
    lens = torch.tensor([0, w.seq_len + 5], dtype=torch.int64, device="cuda")
    cb.cobs_select_blocks_varlen(p.dims, p.q, p.stats, lens, w.seq_len, w.top_k, w.sink_blocks,
                                 w.local_tokens, p.idx, p.idx.shape[-1], p.n_sel, None, p.ws,
                                 p.ws_bytes)
    torch.cuda.synchronize()
    assert p.device_status() == cb.COBS_ERR_DEVICE
