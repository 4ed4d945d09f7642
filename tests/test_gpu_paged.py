"""Paged KV cache on the GPU: page pools plus a block table against the
contiguous calls on the same keys and values (bit-identical), and against the
oracle.

Pages are handed out in a seeded random order with spare pages in the pool;
every row that the table does not map to a token of its sequence (spare
pages, the rows of a last page past its sequence) is NaN, so any read of one
shows up in the results."""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from harness import LSE_ATOL, OUT_ATOL, Problem
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu

W = WORKLOADS
NAN_BITS = 0x7FC0
SENTINEL = 0x1234
CASES = {
    "d128_g4_uniform": (W["single_32k"].scaled(batch=3, q_heads=8, kv_heads=2,
                                                seq_len=4096 + 37), None),
    "d128_g4_ragged": (W["single_32k"].scaled(batch=4, q_heads=8, kv_heads=2,
                                               seq_len=4096 + 37),
                       [4096 + 37, 3500 + 3, 1000 + 1, 130]),
    "d128_g8_r16": (W["build_256k"].scaled(batch=2, seq_len=8192 + 5, append_chunk=0,
                                           decode_steps=1), [8192 + 5, 6000]),
    "d64_g8": (W["tiny_4k"].scaled(batch=3, q_heads=8, kv_heads=1, rank=8, seq_len=2500),
               [2500, 1777, 64]),
}


class Paged:
    def __init__(self, w, lens, seed=11):
        self.p = p = Problem(w)
        self.w = w
        self.ragged = lens is not None
        self.lens = list(lens) if lens is not None else [w.seq_len] * w.batch
        for b, L in enumerate(self.lens):
            p.k[b, :, L:] = NAN_BITS
            p.v[b, :, L:] = NAN_BITS
        self.seq_lens = torch.tensor(self.lens, dtype=torch.int64, device="cuda")
        B = w.block
        nbs = [(L + B - 1) // B for L in self.lens]
        self.n_pages = sum(nbs) + 5                      # spare pages stay unmapped
        # a row length above the blocks addressed, and not a multiple of 4
        self.stride = (w.seq_len + B - 1) // B + 3
        order = np.random.default_rng(seed).permutation(self.n_pages)
        table = np.full((w.batch, self.stride), -1, dtype=np.int32)
        k_pool = torch.full((self.n_pages, w.kv_heads, B, w.head_dim), NAN_BITS,
                            dtype=torch.int16, device="cuda")
        v_pool = torch.full_like(k_pool, NAN_BITS)
        nxt = 0
        for b, L in enumerate(self.lens):
            for j in range(nbs[b]):
                page = int(order[nxt])
                nxt += 1
                table[b, j] = page
                rows = min(B, L - j * B)
                k_pool[page, :, :rows] = p.k[b, :, j * B:j * B + rows]
                v_pool[page, :, :rows] = p.v[b, :, j * B:j * B + rows]
        self.table_np = table
        self.table = torch.from_numpy(table).cuda()
        self.k_pool, self.v_pool = k_pool, v_pool

    # ---- the paged calls --------------------------------------------------------
    def build_stats_paged(self, table, end):
        p = self.p
        cb.cobs_build_block_stats_paged(p.dims, self.k_pool, self.n_pages, table, self.stride,
                                        0, end, p.stats, p.ws, p.ws_bytes)

    def decode_paged(self, table=None):
        p, w = self.p, self.w
        cb.cobs_sparse_decode_paged(p.dims, p.q, self.k_pool, self.v_pool, self.n_pages,
                                    self.table if table is None else table, self.stride,
                                    p.idx, p.n_sel, p.idx.shape[-1],
                                    self.seq_lens if self.ragged else None, w.seq_len,
                                    1.0 / math.sqrt(w.head_dim), p.out, p.lse, p.ws,
                                    p.ws_bytes)

    # ---- the contiguous calls on the same data -----------------------------------
    def build_stats_contiguous(self):
        p, w = self.p, self.w
        d1 = dict(p.dims, batch=1)
        for b, L in enumerate(self.lens):
            if L // w.block:
                cb.cobs_build_block_stats(d1, p.k[b], 0, L // w.block, p.stats[b], p.ws,
                                          p.ws_bytes)

    def select(self):
        p, w = self.p, self.w
        if self.ragged:
            cb.cobs_select_blocks_varlen(p.dims, p.q, p.stats, self.seq_lens, w.seq_len,
                                         w.top_k, w.sink_blocks, w.local_tokens, p.idx,
                                         p.idx.shape[-1], p.n_sel, None, p.ws, p.ws_bytes)
        else:
            p.select(scores=False)

    def decode_contiguous(self):
        p, w = self.p, self.w
        if self.ragged:
            cb.cobs_sparse_decode_varlen(p.dims, p.q, p.k, p.v, p.idx, p.n_sel,
                                         p.idx.shape[-1], self.seq_lens, w.seq_len,
                                         1.0 / math.sqrt(w.head_dim), p.out, p.lse, p.ws,
                                         p.ws_bytes)
        else:
            p.decode()

    def clear_outputs(self):
        self.p.out.fill_(float("nan"))
        self.p.lse.fill_(float("nan"))


@pytest.fixture(scope="module", params=list(CASES))
def pg(request):
    w, lens = CASES[request.param]
    return Paged(w, lens)


def test_paged_stats_match_contiguous(pg):
    """Records of complete blocks are bit-identical; blocks whose table entry
    is negative keep what the buffer held."""
    p, w = pg.p, pg.w
    p.stats.fill_(NAN_BITS)
    pg.build_stats_contiguous()
    ref = p.stats.clone()
    # only complete blocks get a page in this table: the rest must be skipped
    table = pg.table_np.copy()
    for b, L in enumerate(pg.lens):
        table[b, L // w.block:] = -1
    end = max(L // w.block for L in pg.lens)
    p.stats.fill_(SENTINEL)
    pg.build_stats_paged(torch.from_numpy(table).cuda(), end)
    got = p.stats
    for b, L in enumerate(pg.lens):
        nb = L // w.block
        assert torch.equal(got[b, :, :nb], ref[b, :, :nb]), b
        assert bool((got[b, :, nb:] == SENTINEL).all()), b
    assert p.device_status() == 0


def test_paged_decode_matches_contiguous_bitwise(pg):
    p = pg.p
    p.stats.fill_(NAN_BITS)
    pg.build_stats_contiguous()
    pg.select()
    pg.clear_outputs()
    pg.decode_contiguous()
    out_c, lse_c = p.out.clone(), p.lse.clone()
    assert bool(torch.isfinite(out_c).all())
    pg.clear_outputs()
    pg.decode_paged()
    assert torch.equal(p.out, out_c)
    assert torch.equal(p.lse, lse_c)
    assert p.device_status() == 0


def test_paged_decode_against_oracle(pg):
    """The paged decode over the GPU selection against the oracle's attention
    over the same blocks of the contiguous keys and values."""
    p, w = pg.p, pg.w
    p.stats.fill_(NAN_BITS)
    pg.build_stats_contiguous()
    pg.select()
    pg.clear_outputs()
    pg.decode_paged()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    out, lse = p.out.cpu().numpy(), p.lse.cpu().numpy()
    G = w.group
    scale = 1.0 / math.sqrt(w.head_dim)
    for b, L in enumerate(pg.lens):
        for h in range(w.kv_heads):
            sel = idx[b, h, :n[b, h]].astype(np.int64)
            o, l = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h), sel, L,
                                      w.block, scale)
            assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL, (b, h)
            np.testing.assert_allclose(lse[b, h * G:(h + 1) * G], l, atol=LSE_ATOL)
    assert p.device_status() == 0


def test_page_outside_the_pool_is_reported(pg):
    """A selected block whose page lies past the pool is skipped and reported
    through the status word; the call itself succeeds."""
    p, w = pg.p, pg.w
    p.stats.fill_(NAN_BITS)
    pg.build_stats_contiguous()
    pg.select()
    table = pg.table_np.copy()
    tail = (pg.lens[0] + w.block - 1) // w.block - 1
    table[0, tail] = pg.n_pages              # the tail block is always selected
    pg.decode_paged(torch.from_numpy(table).cuda())
    assert p.device_status() == cb.COBS_ERR_DEVICE
    # and the statistics build reports it too
    table[0, 0] = pg.n_pages
    pg.build_stats_paged(torch.from_numpy(table).cuda(), 1)
    assert p.device_status() == cb.COBS_ERR_DEVICE
    assert p.device_status() == 0            # the read cleared it
