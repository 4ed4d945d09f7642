"""Min/max box records and the box selector on the GPU against the oracle.

The box selector is the comparison selector the COBS explainer lists among
the ideas that fall short of COBS (plain-language summary: a block's spread
from the minimum and maximum of its keys).  Reading taken (no formula on the
pages): the box is the per-dimension minimum lo and maximum hi of the block's
keys, a block scores ln n_b + sum_t max(q_t lo_t, q_t hi_t) / sqrt(d) (the
largest logit any point of the box reaches), groups aggregate by log-sum-exp
and the selection is the same top-k + sink + local window as for COBS.

* Records: bit-exact against the oracle's boxes (the minimum and maximum of
  bf16 values are bf16 values), contiguous and paged caches alike.
* Selection over oracle boxes: the oracle's selection up to reported ties,
  scores within the tie tolerance; also at the full 32k batched size.
* End to end: GPU machines, box selection and decode; outputs equal the oracle's
  attention over the oracle's box selection.
"""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from harness import (LSE_ATOL, OUT_ATOL, TIE_RTOL, Problem, _f64_to_bf16_bits, from_dev_bits,
                     selection_mismatch, to_dev)
from workloads import WORKLOADS, bits_to_f64, make_kv_slice, make_queries

pytestmark = pytest.mark.gpu

W = WORKLOADS
CASES = {
    "needles_b2_ragged": W["batched_needles_32k"].scaled(batch=2, seq_len=4096 + 37),
    "g8": W["build_256k"].scaled(seq_len=8192, append_chunk=0, decode_steps=1),
    "g1_d128": W["single_32k"].scaled(q_heads=2, kv_heads=2, seq_len=3000, top_k=5,
                                      local_tokens=100),
    "g2_many_cand": W["single_32k"].scaled(q_heads=4, kv_heads=2, seq_len=80000, top_k=200,
                                           local_tokens=0),
    "d64_g8": W["tiny_4k"].scaled(q_heads=8, kv_heads=1, seq_len=2500, batch=3),
    "d64_g4": W["tiny_4k"],
}


class BoxProblem(Problem):
    def __init__(self, w, **kw):
        super().__init__(w, **kw)
        self.dimsb = dict(self.dims, stats_format=cb.COBS_STATS_BOX)
        assert cb.cobs_stats_record_bytes(self.dimsb) == 4 * w.head_dim
        self.boxes = torch.zeros((w.batch, w.kv_heads, w.cap // w.block, 2, w.head_dim),
                                 dtype=torch.int16, device="cuda")

    def build_boxes(self, begin=0, end=None):
        end = self.w.seq_len // self.w.block if end is None else end
        cb.cobs_build_block_stats(self.dimsb, self.k, begin, end, self.boxes, self.ws,
                                  self.ws_bytes)

    def select_boxes(self):
        w = self.w
        cb.cobs_select_blocks(self.dimsb, self.q, self.boxes, w.seq_len, w.top_k,
                              w.sink_blocks, w.local_tokens, self.idx, self.idx.shape[-1],
                              self.n_sel, self.scores, self.ws, self.ws_bytes)

    def oracle_boxes(self, b, h):
        w = self.w
        return O.build_block_boxes(self.keys(b, h), w.block, 0, w.seq_len // w.block)


@pytest.fixture(scope="module", params=list(CASES))
def bp(request):
    torch.cuda.synchronize()
    return BoxProblem(CASES[request.param], poison="nan")


def test_box_records_are_exact(bp):
    p, w = bp, bp.w
    nfull = w.seq_len // w.block
    p.boxes.fill_(-1)
    p.build_boxes()
    got = from_dev_bits(p.boxes)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            lo, hi = p.oracle_boxes(b, h)
            np.testing.assert_array_equal(bits_to_f64(got[b, h, :nfull, 0]), lo)
            np.testing.assert_array_equal(bits_to_f64(got[b, h, :nfull, 1]), hi)
    # records past the range are untouched
    assert np.all(got[:, :, nfull:] == 0xFFFF)
    assert p.device_status() == 0


def test_box_select_on_oracle_boxes(bp):
    p, w = bp, bp.w
    nfull = w.seq_len // w.block
    orc = {}
    for b in range(w.batch):
        for h in range(w.kv_heads):
            lo, hi = p.oracle_boxes(b, h)
            p.boxes[b, h, :nfull, 0] = to_dev(_f64_to_bf16_bits(lo))
            p.boxes[b, h, :nfull, 1] = to_dev(_f64_to_bf16_bits(hi))
            orc[(b, h)] = O.select_from_boxes(p.q_group(b, h), lo, hi, w.seq_len, w.block,
                                              w.top_k, w.sink_blocks, w.local_tokens)
    p.select_boxes()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    scores = p.scores.cpu().numpy()
    _, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
    for (b, h), (sel, s) in orc.items():
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0)
        assert n[b, h] == len(sel)
        assert selection_mismatch(got, sel, s, w) == [], (b, h)
        if c1 > c0:
            np.testing.assert_allclose(scores[b, h, c0:c1], s[c0:c1], rtol=0,
                                       atol=TIE_RTOL * max(1, np.max(np.abs(s))))
    assert p.device_status() == 0


def test_box_end_to_end(bp):
    p, w = bp, bp.w
    p.build_boxes()
    p.select_boxes()
    p.decode()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    out, lse = p.out.cpu().numpy(), p.lse.cpu().numpy()
    G = w.group
    scale = 1 / math.sqrt(w.head_dim)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            lo, hi = p.oracle_boxes(b, h)
            sel, s = O.select_from_boxes(p.q_group(b, h), lo, hi, w.seq_len, w.block, w.top_k,
                                         w.sink_blocks, w.local_tokens)
            got = idx[b, h, :n[b, h]]
            # the records are exact, so the selections agree up to score ties
            assert selection_mismatch(got, sel, s, w) == [], (b, h)
            o, l = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h),
                                      got.astype(np.int64), w.seq_len, w.block, scale)
            assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL
            np.testing.assert_allclose(lse[b, h * G:(h + 1) * G], l, atol=LSE_ATOL)
    assert p.device_status() == 0


def test_box_records_paged_match_contiguous():
    w = W["single_32k"].scaled(batch=2, q_heads=8, kv_heads=2, seq_len=4096 + 64 * 3)
    p = BoxProblem(w)
    nb = w.seq_len // w.block
    p.build_boxes()
    want = p.boxes.clone()
    # pages in a seeded random order, one spare page, an unmapped block (-1)
    rng = np.random.default_rng(3)
    n_pages = w.batch * nb + 1
    perm = rng.permutation(n_pages)[:w.batch * nb].reshape(w.batch, nb).astype(np.int32)
    pool = torch.full((n_pages, w.kv_heads, w.block, w.head_dim), -1, dtype=torch.int16,
                      device="cuda")
    for b in range(w.batch):
        for j in range(nb):
            pool[int(perm[b, j])] = p.k[b, :, j * 64:(j + 1) * 64]
    table = torch.from_numpy(perm.copy()).cuda()
    table[1, 5] = -1
    got = torch.zeros_like(p.boxes)
    got[1, :, 5] = 7
    cb.cobs_build_block_stats_paged(p.dimsb, pool, n_pages, table, nb, 0, nb, got, p.ws,
                                    p.ws_bytes)
    torch.cuda.synchronize()
    assert torch.all(got[1, :, 5] == 7)            # a block without a page keeps its record
    got[1, :, 5] = want[1, :, 5]
    assert torch.equal(got, want)
    assert p.device_status() == 0


def test_box_select_at_full_size():
    """Box selection in the launch the full 32k batched workload gets (64
    records per 128-row tile, every pair's 503 candidates in one CTA), on
    sampled pairs with the oracle's boxes uploaded."""
    w = W["batched_needles_32k"]
    dims = dict(batch=w.batch, num_q_heads=w.q_heads, num_kv_heads=w.kv_heads,
                head_dim=w.head_dim, block_size=w.block, rank=w.rank, capacity_tokens=w.cap,
                stats_format=cb.COBS_STATS_BOX)
    q_bits = make_queries(w)
    q = to_dev(q_bits)
    nb_cap, nfull = w.cap // w.block, w.seq_len // w.block
    boxes = torch.zeros((w.batch, w.kv_heads, nb_cap, 2, w.head_dim), dtype=torch.int16,
                        device="cuda")
    nsm = cb.cobs_selected_capacity(dims, w.top_k, w.sink_blocks, w.local_tokens)
    idx = torch.zeros((w.batch, w.kv_heads, nsm), dtype=torch.int32, device="cuda")
    n_sel = torch.zeros((w.batch, w.kv_heads), dtype=torch.int32, device="cuda")
    ws_bytes = cb.cobs_workspace_bytes(dims, w.top_k, w.sink_blocks, w.local_tokens)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    cb.cobs_workspace_init(ws, ws_bytes)
    pairs = [(0, 0), (13, 4), (31, 7)]
    orc = {}
    G = w.group
    for (b, h) in pairs:
        kb, _ = make_kv_slice(w, b, h, q_bits)
        lo, hi = O.build_block_boxes(bits_to_f64(kb), w.block, 0, nfull)
        boxes[b, h, :nfull, 0] = to_dev(_f64_to_bf16_bits(lo))
        boxes[b, h, :nfull, 1] = to_dev(_f64_to_bf16_bits(hi))
        orc[(b, h)] = O.select_from_boxes(bits_to_f64(q_bits[b, h * G:(h + 1) * G]), lo, hi,
                                          w.seq_len, w.block, w.top_k, w.sink_blocks,
                                          w.local_tokens)
    cb.cobs_select_blocks(dims, q, boxes, w.seq_len, w.top_k, w.sink_blocks, w.local_tokens,
                          idx, nsm, n_sel, None, ws, ws_bytes)
    idx_h, n_h = idx.cpu().numpy(), n_sel.cpu().numpy()
    for (b, h), (sel, s) in orc.items():
        got = idx_h[b, h, :n_h[b, h]]
        assert len(got) == len(sel) and selection_mismatch(got, sel, s, w) == [], (b, h)
    assert cb.cobs_read_device_status(ws, ws_bytes) == 0
