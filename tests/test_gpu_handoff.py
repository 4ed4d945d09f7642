"""cobs_select_and_decode: where every (batch, kv-head) is one decode chunk,
the selection hands each pair to the decode as soon as its list is written,
and the decode takes the pairs in the order they finish; otherwise (pairs
split into chunks and merged by the second kernel, head_dim 64) the kernels
run in turn.  Per pair the arithmetic is that of the two separate calls, so
the lists, counts, scores, outputs and log-sum-exps must be bit-identical to
cobs_select_blocks followed by cobs_sparse_decode, over repeated calls that
alternate with the separate calls on one workspace (the ready list's epoch
and count must be left ready for the next use).  The outputs are also checked
against the oracle's attention over the lists."""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from harness import LSE_ATOL, OUT_ATOL, Problem
from workloads import WORKLOADS as W

pytestmark = pytest.mark.gpu

CASES = {
    # 256 pairs: one decode chunk each (handed over)
    "pairs256_whole": W["batched_needles_32k"].scaled(seq_len=8192 + 21),
    # 512 pairs: more pairs than resident decode CTAs (handed over, CTAs
    # taking several pairs)
    "pairs512_whole": W["batched_needles_32k"].scaled(batch=64, seq_len=4096),
    # 64 pairs: split into chunks, merged
    "pairs64_split": W["batched_needles_32k"].scaled(batch=8, seq_len=8192),
    # 4 pairs, G = 4: many chunks per pair
    "pairs4_g4": W["single_32k"].scaled(seq_len=16384 + 64 * 3),
    # 8 pairs, G = 8, r = 16, top-64
    "pairs8_g8_r16": W["build_256k"].scaled(seq_len=16384, append_chunk=0, decode_steps=1),
    # head_dim 64: the two kernels in turn
    "d64": W["tiny_4k"].scaled(batch=3, seq_len=4096 - 37),
}


def fused(p, scores):
    w = p.w
    cb.cobs_select_and_decode(p.dims, p.q, p.stats, p.k, p.v, w.seq_len, w.top_k,
                              w.sink_blocks, w.local_tokens, 1.0 / math.sqrt(w.head_dim),
                              p.idx, p.idx.shape[-1], p.n_sel, scores, p.out, p.lse, p.ws,
                              p.ws_bytes)


def snapshot(p):
    torch.cuda.synchronize()
    return [t.clone() for t in (p.idx, p.n_sel, p.scores, p.out, p.lse)]


@pytest.mark.parametrize("name", list(CASES))
def test_fused_equals_separate_calls(name):
    w = CASES[name]
    p = Problem(w, poison="nan")
    p.build_stats()
    p.select()
    p.decode()
    want = snapshot(p)
    for rep in range(3):   # epochs 1..3, with separate calls in between
        for t in (p.idx, p.out, p.lse, p.scores):
            t.fill_(-7 if t.dtype == torch.int32 else float("nan"))
        p.n_sel.zero_()
        fused(p, p.scores)
        got = snapshot(p)
        for a, b, what in zip(got, want, ("idx", "n_sel", "scores", "out", "lse")):
            if what == "idx":   # rows past n_sel are not written by either path
                n = want[1].cpu().numpy()
                ga, wa = a.cpu().numpy(), b.cpu().numpy()
                for bb in range(w.batch):
                    for hh in range(w.kv_heads):
                        k = n[bb, hh]
                        assert np.array_equal(ga[bb, hh, :k], wa[bb, hh, :k]), (rep, bb, hh)
            elif what == "scores":
                _, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks,
                                              w.local_tokens)
                assert torch.equal(a[:, :, c0:c1], b[:, :, c0:c1]), rep
            else:
                assert torch.equal(a, b), (rep, what)
        assert p.device_status() == 0, rep
        p.select()          # the separate calls still work on the same workspace
        p.decode()
        torch.cuda.synchronize()
        assert torch.equal(p.out, want[3]) and torch.equal(p.lse, want[4]), rep
    # and against the oracle's attention over the lists, on sampled pairs
    out, lse = p.out.cpu().numpy(), p.lse.cpu().numpy()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    G = w.group
    for (b, h) in sorted({(0, 0), (w.batch - 1, w.kv_heads - 1)}):
        o, l = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h),
                                  idx[b, h, :n[b, h]].astype(np.int64), w.seq_len, w.block,
                                  1.0 / math.sqrt(w.head_dim))
        assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL, (b, h)
        np.testing.assert_allclose(lse[b, h * G:(h + 1) * G], l, atol=LSE_ATOL)
    assert p.device_status() == 0


def test_fused_in_a_cuda_graph():
    """Replayed from a CUDA graph (as the bench drives it), repeatedly: the
    same results as the separate calls every time."""
    w = CASES["pairs256_whole"]
    p = Problem(w)
    p.build_stats()
    p.select()
    p.decode()
    want = snapshot(p)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        fused(p, None)      # warm-up outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            cb.cobs_select_and_decode(p.dims, p.q, p.stats, p.k, p.v, w.seq_len, w.top_k,
                                      w.sink_blocks, w.local_tokens,
                                      1.0 / math.sqrt(w.head_dim), p.idx, p.idx.shape[-1],
                                      p.n_sel, None, p.out, p.lse, p.ws, p.ws_bytes,
                                      s.cuda_stream)
    for rep in range(5):
        p.out.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(p.out, want[3]) and torch.equal(p.lse, want[4]), rep
    assert p.device_status() == 0
