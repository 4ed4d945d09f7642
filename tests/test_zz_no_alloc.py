"""The allocation-free decode entry point against the workspace one and the oracle.

cobs_sparse_decode_no_alloc exists for callers that cannot hand the library
device memory (their framework owns every device allocation, or they run where
allocating is forbidden or too slow); it keeps its split-K scratch and its
status word in the library's own fixed device array instead.  Its results must
match cobs_sparse_decode on the same inputs, call after call, since the scratch
is shared and keeps the previous call's contents, and they must match the
oracle's attention over the same block lists.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.  It builds its own inputs, so
it passes alone in a fresh process as well as after the other tests.
"""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from harness import LSE_ATOL, OUT_ATOL, Problem
from workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def _lists(p, seed):
    """Random block lists of varying lengths (unordered) for every pair."""
    w = p.w
    rng = np.random.default_rng(seed)
    nbs = -(-w.seq_len // w.block)
    idx = torch.full_like(p.idx, -1)
    n = torch.zeros_like(p.n_sel)
    lists = {}
    for b in range(w.batch):
        for h in range(w.kv_heads):
            k = int(rng.integers(1, min(p.nsm, nbs) + 1))
            sel = rng.choice(nbs, size=k, replace=False).astype(np.int32)
            idx[b, h, :k] = torch.from_numpy(sel).cuda()
            n[b, h] = k
            lists[(b, h)] = sel
    return idx, n, lists


@pytest.mark.parametrize("name,kw", [
    ("batched_needles_32k", dict(batch=4, seq_len=8192 + 21)),
    ("build_256k", dict(seq_len=16384, append_chunk=0, decode_steps=1)),
    ("tiny_4k", dict(batch=3, seq_len=4096 - 37)),          # head_dim 64 kernel
])
def test_no_alloc_decode_matches_workspace_decode_twice(name, kw):
    w = WORKLOADS[name].scaled(**kw)
    p = Problem(w, poison="nan")
    scale = 1.0 / math.sqrt(w.head_dim)
    assert cb.cobs_no_alloc_read_status() in (0, cb.COBS_ERR_DEVICE)   # clear leftovers
    G = w.group
    for call, seed in enumerate((11, 12)):          # two calls in a row
        idx, n, lists = _lists(p, seed)
        cb.cobs_sparse_decode(p.dims, p.q, p.k, p.v, idx, n, p.nsm, w.seq_len, scale,
                              p.out, p.lse, p.ws, p.ws_bytes)
        torch.cuda.synchronize()
        want_out, want_lse = p.out.clone(), p.lse.clone()
        out = torch.full_like(p.out, float("nan"))
        lse = torch.full_like(p.lse, float("nan"))
        cb.cobs_sparse_decode_no_alloc(p.dims, p.q, p.k, p.v, idx, n, p.nsm, w.seq_len,
                                       scale, out, lse)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all() and torch.isfinite(lse).all(), call
        assert (out - want_out).abs().max().item() <= OUT_ATOL, call
        assert (lse - want_lse).abs().max().item() <= LSE_ATOL, call
        # the oracle's exact attention over the same lists, on sampled pairs
        out_h, lse_h = out.cpu().numpy(), lse.cpu().numpy()
        for (b, h) in sorted({(0, 0), (w.batch - 1, w.kv_heads - 1)}):
            o, l = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h),
                                      np.sort(lists[(b, h)]), w.seq_len, w.block, scale)
            assert np.max(np.abs(out_h[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL, (call, b, h)
            assert np.max(np.abs(lse_h[b, h * G:(h + 1) * G] - l)) <= LSE_ATOL, (call, b, h)
        assert cb.cobs_no_alloc_read_status() == 0, call
    assert p.device_status() == 0


@pytest.mark.parametrize("name", ["batched_needles_32k", "tiny_4k"])
def test_no_alloc_reports_device_errors_in_its_own_status_word(name):
    # a block index past the sequence is skipped and reported: the fixed
    # array's status word keeps the report until it is read, then reads clean
    w = WORKLOADS[name].scaled(batch=2, seq_len=2048)
    p = Problem(w)
    scale = 1.0 / math.sqrt(w.head_dim)
    cb.cobs_no_alloc_read_status()
    idx = torch.zeros_like(p.idx)
    n = torch.ones_like(p.n_sel)
    idx[1, 0, 0] = w.seq_len // w.block + 3          # outside [0, ceil(seq_len / 64))
    out = torch.zeros_like(p.out)
    lse = torch.zeros_like(p.lse)
    cb.cobs_sparse_decode_no_alloc(p.dims, p.q, p.k, p.v, idx, n, p.nsm, w.seq_len, scale,
                                   out, lse)
    torch.cuda.synchronize()
    assert cb.cobs_no_alloc_read_status() == cb.COBS_ERR_DEVICE
    assert cb.cobs_no_alloc_read_status() == 0       # cleared by the read
    idx[1, 0, 0] = 0
    cb.cobs_sparse_decode_no_alloc(p.dims, p.q, p.k, p.v, idx, n, p.nsm, w.seq_len, scale,
                                   out, lse)
    torch.cuda.synchronize()
    assert cb.cobs_no_alloc_read_status() == 0


def test_no_alloc_rejects_problems_beyond_its_fixed_scratch():
    # 4096 sequences x 64 query heads at d = 128 need far more than 16 MiB of
    # split partials; the call must refuse before touching any memory
    dims = dict(batch=4096, num_q_heads=64, num_kv_heads=8, head_dim=128, block_size=64,
                rank=8, capacity_tokens=64)
    fake = 1 << 20
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_sparse_decode_no_alloc(dims, fake, fake, fake, fake, fake, 64, 64, 0.1,
                                       fake, fake)
    assert e.value.status == cb.COBS_ERR_WORKSPACE
    assert "fixed" in cb.cobs_last_error()
