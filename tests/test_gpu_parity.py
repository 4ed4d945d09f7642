"""GPU parity on small and ragged cases: each CUDA entry point, called through
the C ABI, against the oracle element by element.  Sizes span several tiles
(blocks, splits, chunks) and a ragged tail; the full-size workloads are in
test_gpu_fullsize.py."""

import math

import numpy as np
import pytest
import torch

import oracle.cobs_oracle as O
from harness import (ENERGY_RTOL, LSE_ATOL, OUT_ATOL, PROJ_RTOL, TIE_RTOL, Problem,
                     block_is_gapped, explain_selection, from_dev_bits, score_change_bound,
                     selection_mismatch, stats_errors, to_dev)
from workloads import WORKLOADS, bits_to_f64, to_bf16_bits

pytestmark = pytest.mark.gpu

W = WORKLOADS
CASES = {
    "tiny_4k": W["tiny_4k"],
    "single_ragged": W["single_32k"].scaled(seq_len=4096 + 37),
    "needles_b2": W["batched_needles_32k"].scaled(batch=2, seq_len=4096),
    "long_b2": W["long_128k"].scaled(batch=2, seq_len=8192 + 64 * 3 + 5),
    "g8_r16": W["build_256k"].scaled(seq_len=8192, append_chunk=0, decode_steps=1),
    "g1_d128": W["single_32k"].scaled(q_heads=2, kv_heads=2, seq_len=3000, top_k=5,
                                      local_tokens=100),
    "g2_r0": W["single_32k"].scaled(q_heads=4, kv_heads=2, seq_len=2048 + 1, rank=0),
    "d64_g8_r8": W["tiny_4k"].scaled(q_heads=8, kv_heads=1, rank=8, seq_len=2500,
                                     batch=3),
    "d64_g2_r16": W["tiny_4k"].scaled(q_heads=4, kv_heads=2, rank=16, seq_len=1111,
                                      local_tokens=0),
}


@pytest.fixture(scope="module", params=list(CASES))
def prob(request):
    torch.cuda.synchronize()
    return Problem(CASES[request.param], poison="nan")


def oracle_selection(p, b, h, recs=None):
    w = p.w
    recs = p.oracle_records(b, h) if recs is None else recs
    return O.select_from_records(p.q_group(b, h), recs, w.seq_len, w.block, w.top_k,
                                 w.sink_blocks, w.local_tokens)


def upload_idx(p, lists):
    idx = torch.full_like(p.idx, -3)
    n = torch.zeros_like(p.n_sel)
    for (b, h), sel in lists.items():
        idx[b, h, :len(sel)] = torch.tensor(np.asarray(sel, np.int32), device="cuda")
        n[b, h] = len(sel)
    return idx, n


def check_decode(p, lists):
    w = p.w
    idx, n = upload_idx(p, lists)
    p.decode(idx=idx, n_sel=n)
    out = p.out.cpu().numpy()
    lse = p.lse.cpu().numpy()
    scale = 1 / math.sqrt(w.head_dim)
    G = w.group
    worst = 0.0
    for (b, h), sel in lists.items():
        o, l = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h), sel,
                                  w.seq_len, w.block, scale)
        e = np.max(np.abs(out[b, h * G:(h + 1) * G] - o))
        worst = max(worst, e)
        assert e <= OUT_ATOL, ((b, h), e)
        np.testing.assert_allclose(lse[b, h * G:(h + 1) * G], l, atol=LSE_ATOL)
    assert p.device_status() == 0
    return worst


def test_decode_on_oracle_selection(prob):
    p, w = prob, prob.w
    lists = {(b, h): oracle_selection(p, b, h)[0]
             for b in range(w.batch) for h in range(w.kv_heads)}
    check_decode(p, lists)


def test_decode_random_lists_varying_lengths(prob):
    p, w = prob, prob.w
    rng = np.random.default_rng(5)
    nbs = -(-w.seq_len // w.block)
    lists = {}
    for b in range(w.batch):
        for h in range(w.kv_heads):
            n = int(rng.integers(1, min(p.nsm, nbs) + 1))
            lists[(b, h)] = rng.choice(nbs, size=n, replace=False)   # unordered
    check_decode(p, lists)


def test_decode_with_every_block_is_dense_attention(prob):
    p, w = prob, prob.w
    nbs = -(-w.seq_len // w.block)
    idx = torch.arange(nbs, dtype=torch.int32, device="cuda").expand(
        w.batch, w.kv_heads, nbs).contiguous()
    n = torch.full((w.batch, w.kv_heads), nbs, dtype=torch.int32, device="cuda")
    # this stride exceeds the workspace the problem sized; use a larger one
    import block_sparse_long_cobs_b200 as cb
    dims = dict(p.dims)
    ws_bytes = cb.cobs_workspace_bytes(dims, nbs, 0, 0)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
    cb.cobs_sparse_decode(dims, p.q, p.k, p.v, idx, n, nbs, w.seq_len,
                          1 / math.sqrt(w.head_dim), p.out, p.lse, ws, ws_bytes)
    out, lse = p.out.cpu().numpy(), p.lse.cpu().numpy()
    G = w.group
    for b in range(w.batch):
        for h in range(w.kv_heads):
            o, l = O.dense_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h),
                                     w.seq_len, 1 / math.sqrt(w.head_dim))
            assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL
            np.testing.assert_allclose(lse[b, h * G:(h + 1) * G], l, atol=LSE_ATOL)
    assert cb.cobs_read_device_status(ws, ws_bytes) == 0


def test_select_on_oracle_stats(prob):
    p, w = prob, prob.w
    orc = {}
    for b in range(w.batch):
        for h in range(w.kv_heads):
            recs = p.oracle_records(b, h)
            p.upload_records(b, h, recs)
            orc[(b, h)] = oracle_selection(p, b, h, recs)
    p.select()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    scores = p.scores.cpu().numpy()
    forced, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
    for (b, h), (sel, s) in orc.items():
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0)
        assert n[b, h] == len(sel)
        assert selection_mismatch(got, sel, s, w) == []
        if c1 > c0:
            np.testing.assert_allclose(scores[b, h, c0:c1], s[c0:c1],
                                       rtol=0, atol=TIE_RTOL * max(1, np.max(np.abs(s))))
    assert p.device_status() == 0


def test_stats_build(prob):
    p, w = prob, prob.w
    p.build_stats()
    torch.cuda.synchronize()
    st = from_dev_bits(p.stats)
    nfull = w.seq_len // w.block
    worst_proj, worst_energy = 0.0, 1.0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            keys = p.keys(b, h)
            orc = p.oracle_records(b, h)
            gpu = bits_to_f64(st[b, h, :nfull])
            for j in range(nfull):
                mu_ok, rel, energy = stats_errors(gpu[j], orc[j],
                                                  keys[j * w.block:(j + 1) * w.block],
                                                  w.rank)
                assert mu_ok, (b, h, j)
                if rel is not None:
                    worst_proj = max(worst_proj, rel)
                    assert rel <= PROJ_RTOL, (b, h, j, rel)
                worst_energy = min(worst_energy, energy)
                assert energy >= 1 - ENERGY_RTOL, (b, h, j, energy)
    # blocks past the range are untouched
    if nfull < st.shape[2]:
        assert np.all(st[:, :, nfull:] == 0)
    assert p.device_status() == 0


def test_end_to_end_pipeline(prob):
    """GPU stats, selection and decode against the oracle on every pair: each
    selection flip explained by the records (explain_selection), outputs equal
    to the oracle's attention over the GPU's selection."""
    p, w = prob, prob.w
    p.build_stats()
    p.select()
    p.decode()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    out = p.out.cpu().numpy()
    st = from_dev_bits(p.stats)
    G = w.group
    scale = 1 / math.sqrt(w.head_dim)
    nfull = w.seq_len // w.block
    flips = 0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            recs = p.oracle_records(b, h)
            got = idx[b, h, :n[b, h]]
            nd, _, rows = explain_selection(w, p.q_group(b, h), got,
                                            bits_to_f64(st[b, h, :nfull]), recs)
            flips += nd > 0
            keys = p.keys(b, h)
            for (j, _, _, change) in rows:
                if block_is_gapped(keys[j * 64:(j + 1) * 64], w.rank):
                    assert change <= score_change_bound(p.q_group(b, h), recs[j], w.rank)
            o, _ = O.sparse_attention(p.q_group(b, h), keys, p.values(b, h),
                                      got.astype(np.int64), w.seq_len, w.block, scale)
            assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL
    print(f"end-to-end selections differing from the oracle's: {flips} of "
          f"{w.batch * w.kv_heads} pairs (each explained by its records)")
    assert p.device_status() == 0


def test_repeat_and_graph_replay_are_stable(prob):
    p, w = prob, prob.w
    p.build_stats()
    p.select()
    p.decode()
    torch.cuda.synchronize()
    ref = (p.idx.clone(), p.n_sel.clone(), p.out.clone(), p.lse.clone(), p.stats.clone())
    for _ in range(2):
        p.build_stats()
        p.select()
        p.decode()
    torch.cuda.synchronize()
    for a, b in zip(ref, (p.idx, p.n_sel, p.out, p.lse, p.stats)):
        assert torch.equal(a, b)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            import block_sparse_long_cobs_b200 as cb
            cb.cobs_select_blocks(p.dims, p.q, p.stats, w.seq_len, w.top_k, w.sink_blocks,
                                  w.local_tokens, p.idx, p.nsm, p.n_sel, None, p.ws,
                                  p.ws_bytes, stream=s)
            cb.cobs_sparse_decode(p.dims, p.q, p.k, p.v, p.idx, p.n_sel, p.nsm, w.seq_len,
                                  1 / math.sqrt(w.head_dim), p.out, p.lse, p.ws,
                                  p.ws_bytes, stream=s)
    p.out.zero_()
    p.idx.fill_(-1)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    n = p.n_sel.cpu().numpy()
    a_idx, b_idx = ref[0].cpu().numpy(), p.idx.cpu().numpy()
    for b in range(w.batch):
        for h in range(w.kv_heads):
            assert list(a_idx[b, h, :n[b, h]]) == list(b_idx[b, h, :n[b, h]])
    assert torch.equal(ref[2], p.out) and torch.equal(ref[1], p.n_sel)
    del g
    assert p.device_status() == 0


# ---------------------------------------------------------------------------
# selection edge cases on oracle stats
# ---------------------------------------------------------------------------

EDGE = W["single_32k"].scaled(seq_len=2048 + 10, batch=2, q_heads=8, kv_heads=2)


@pytest.fixture(scope="module")
def edge():
    p = Problem(EDGE)
    recs = {}
    for b in range(EDGE.batch):
        for h in range(EDGE.kv_heads):
            r = p.oracle_records(b, h)
            if (b, h) == (1, 1):
                # exact ties: copy block 3's record onto blocks 9, 12 and 20
                r[[9, 12, 20]] = r[3]
            recs[(b, h)] = r
            p.upload_records(b, h, r)
    return p, recs


@pytest.mark.parametrize("seq_len,top_k,sink,local", [
    (2048 + 10, 4, 1, 512),      # ragged tail, normal
    (2048 + 10, 100, 1, 512),    # top_k >= candidates -> every block
    (2048 + 10, 0, 1, 512),      # no top-k: forced blocks only
    (2048, 6, 1, 0),             # no local window, block-aligned
    (2000, 6, 1, 0),             # no local window, partial tail forced
    (300, 6, 1, 512),            # window covers the whole sequence
    (2048 + 10, 6, 0, 64),       # no sink
    (2048 + 10, 6, 3, 64),       # three sink blocks
    (64 * 5, 2, 4, 100),         # sink reaches into the window
    (1, 3, 1, 1),                # one token
])
def test_select_edge_cases(edge, seq_len, top_k, sink, local):
    p, recs = edge
    w = EDGE.scaled(seq_len=seq_len, top_k=top_k, sink_blocks=sink, local_tokens=local)
    import block_sparse_long_cobs_b200 as cb
    nsm = cb.cobs_selected_capacity(p.dims, top_k, sink, local)
    p.idx = torch.full((w.batch, w.kv_heads, nsm), -9, dtype=torch.int32, device="cuda")
    p.select(seq_len=seq_len, top_k=top_k, sink=sink, local=local)
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    for (b, h), r in recs.items():
        sel, s = O.select_from_records(p.q_group(b, h), r, seq_len, w.block, top_k, sink,
                                       local)
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0)
        assert len(got) == len(sel)
        if (b, h) == (1, 1):
            assert list(got) == list(sel)     # exact ties broken by index
        else:
            assert selection_mismatch(got, sel, s, w, seq_len) == []
    assert p.device_status() == 0


def test_planted_spectrum_blocks():
    """Blocks with an exactly known covariance: U U^T must reproduce it."""
    w = W["single_32k"].scaled(seq_len=64 * 8, batch=1, q_heads=4, kv_heads=1, rank=8)
    p = Problem(w)
    rng = np.random.default_rng(3)
    from test_oracle_pins import planted_block
    kb = p.k_bits.copy()
    want = []
    for j in range(8):
        lam = np.sort(rng.uniform(0.2, 3.0, size=6))[::-1] * (1 + j)
        mu = 0.3 * rng.standard_normal(w.head_dim)
        keys, v = planted_block(64, w.head_dim, lam, mu, seed=j)
        from workloads import to_bf16_bits
        kb[0, 0, j * 64:(j + 1) * 64] = to_bf16_bits(keys)
        want.append(bits_to_f64(to_bf16_bits(keys)))
    p.k = to_dev(kb)
    p.build_stats()
    st = bits_to_f64(from_dev_bits(p.stats))
    for j in range(8):
        orc = O.block_record(want[j], w.rank)
        mu_ok, rel, energy = stats_errors(st[0, 0, j], orc, want[j], w.rank)
        assert mu_ok and energy >= 1 - ENERGY_RTOL
        assert rel is None or rel <= PROJ_RTOL


@pytest.mark.parametrize("seq_len,top_k", [
    (16384 + 5, 127), (16384 + 5, 128), (16384 + 5, 200),   # <= 1024 candidates
    (80000 + 5, 100), (80000 + 5, 300),                       # grouped candidates
])
def test_select_large_top_k(seq_len, top_k):
    """top_k below, at and above the 128 threads' worth of maxima, over fewer
    and more than 1024 candidates (the grouped bound): the selection must be
    exact; planted exact ties must still be broken by the lower block index."""
    w = W["single_32k"].scaled(seq_len=seq_len, batch=1, q_heads=8, kv_heads=2,
                               top_k=top_k)
    p = Problem(w)
    recs = {}
    for h in range(w.kv_heads):
        r = p.oracle_records(0, h)
        if h == 1:
            r[[50, 60, 70, 200]] = r[40]
        recs[(0, h)] = r
        p.upload_records(0, h, r)
    p.select()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    for (b, h), r in recs.items():
        sel, s = O.select_from_records(p.q_group(b, h), r, w.seq_len, w.block, w.top_k,
                                       w.sink_blocks, w.local_tokens)
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0)
        assert len(got) == len(sel)
        if h == 1:
            assert list(got) == list(sel)
        else:
            assert selection_mismatch(got, sel, s, w) == []
    assert p.device_status() == 0


@pytest.mark.parametrize("top_k", [8, 100])
def test_select_too_many_candidates_to_stage(top_k):
    """16383 candidate blocks at head_dim 64 (a 1M-token cache): their scores
    do not fit beside the top-k's work arrays in the 48 KB record ring, so the
    top-k reads them from global memory instead of shared memory.  Records
    are seeded random bf16 values (the statistics build is not under test);
    the selection must equal the oracle's over the same records, and planted
    exact ties must go to the lower block index."""
    w = W["tiny_4k"].scaled(seq_len=1 << 20, top_k=top_k)
    p = Problem(w)
    rng = np.random.default_rng(17)
    nfull = w.seq_len // w.block
    shape = (nfull, 1 + w.rank, w.head_dim)
    recs = rng.standard_normal(shape) * np.array([0.5] + [0.3] * w.rank)[None, :, None]
    recs = bits_to_f64(to_bf16_bits(recs))
    tied = [700, 900, 5000, 12000]
    recs[tied[1:]] = recs[tied[0]]                 # exact ties: equal scores
    p.upload_records(0, 0, recs)
    p.select()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    sel, s = O.select_from_records(p.q_group(0, 0), recs, w.seq_len, w.block, w.top_k,
                                   w.sink_blocks, w.local_tokens)
    got = idx[0, 0, :n[0, 0]]
    assert np.all(np.diff(got) > 0)
    assert len(got) == len(sel)
    assert selection_mismatch(got, sel, s, w) == []
    want, have = set(sel.tolist()), set(got.tolist())
    assert [t in have for t in tied] == [t in want for t in tied]   # lower index first
    assert p.device_status() == 0
