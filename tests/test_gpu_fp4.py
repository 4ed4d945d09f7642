"""FP4 block records (COBS explainer §2.3, quantisation: U in scaled FP4 E2M1,
mu in bf16) on the GPU against the oracle.

* Selection over oracle-built FP4 records: the same blocks as the oracle's
  selection from those records (up to reported score ties), scores within the
  tie tolerance.
* The statistics build writing FP4: mu bit-identical to the bf16 build; every
  scale exponent and code equal to the oracle's quantisation of the exact
  factor, except where the oracle's own value sits within a small margin of a
  rounding boundary (the GPU quantises its fp32 factor, the oracle the fp64
  one) -- there the two codes must be the neighbours across that boundary.
  Columns are compared where the eigenvalue gaps fix them (up to sign).
* End to end: GPU FP4 statistics, selection and decode; outputs match the
  oracle's attention over the selected blocks, selection flips are counted.
"""

import math

import numpy as np
import pytest
import torch

import block_sparse_long_cobs_b200 as cb
import oracle.cobs_oracle as O
from harness import (OUT_ATOL, PROJ_RTOL, TIE_RTOL, Fp4Problem, explain_selection,
                     from_dev_bits, selection_mismatch, to_dev, unpack_fp4_records)
from workloads import WORKLOADS, bits_to_f64, to_bf16_bits

pytestmark = pytest.mark.gpu

W = WORKLOADS
CASES = {
    "needles_b2_r8": W["batched_needles_32k"].scaled(batch=2, seq_len=4096 + 37),
    "g8_r16": W["build_256k"].scaled(seq_len=8192, append_chunk=0, decode_steps=1),
    "g1_r1": W["single_32k"].scaled(q_heads=2, kv_heads=2, seq_len=3000, rank=1, top_k=5,
                                    local_tokens=100),
    "d64_g8_r8": W["tiny_4k"].scaled(q_heads=8, kv_heads=1, rank=8, seq_len=2500, batch=3),
    "d64_g2_r4": W["tiny_4k"].scaled(q_heads=4, kv_heads=2, rank=4, seq_len=1111,
                                     local_tokens=0),
}
MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
NEAR = 5e-2          # |x - midpoint| in units of the group scale counted as a boundary case
GAP_COLUMN = 1.05    # eigenvalue ratio to both neighbours that fixes a column


@pytest.fixture(scope="module", params=list(CASES))
def fp(request):
    torch.cuda.synchronize()
    return Fp4Problem(CASES[request.param], poison="nan")


def oracle_selection4(p, b, h, parts):
    w = p.w
    recs = O.fp4_record_values(*parts)
    return O.select_from_records(p.q_group(b, h), recs, w.seq_len, w.block, w.top_k,
                                 w.sink_blocks, w.local_tokens)


def test_select_on_oracle_fp4_records(fp):
    p, w = fp, fp.w
    orc = {}
    for b in range(w.batch):
        for h in range(w.kv_heads):
            parts = p.oracle_records4(b, h)
            p.upload_records4(b, h, parts)
            orc[(b, h)] = oracle_selection4(p, b, h, parts)
    p.select4()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    scores = p.scores.cpu().numpy()
    forced, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
    for (b, h), (sel, s) in orc.items():
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0)
        assert n[b, h] == len(sel)
        assert selection_mismatch(got, sel, s, w) == [], (b, h)
        if c1 > c0:
            np.testing.assert_allclose(scores[b, h, c0:c1], s[c0:c1],
                                       rtol=0, atol=TIE_RTOL * max(1, np.max(np.abs(s))))
    assert p.device_status() == 0


def check_fp4_block(mu_g, codes_g, sb_g, pad_g, keys, rank, stats):
    """One GPU FP4 record against the oracle's quantisation of the exact factor."""
    mu_o, codes_o, sb_o = O.block_record_fp4(keys, rank)
    assert np.all(pad_g == 0)
    _, sigma = O.block_moments(keys)
    u_o, _ = O.covariance_factor(sigma, rank)
    lam = np.sort(np.linalg.eigvalsh(sigma))[::-1]
    d = keys.shape[1]
    # the whole factor, rotation-free: |U^ U^T - U U^T|_F within the rounding
    # bound of the codes (half a grid step each, from the GPU's own scales)
    # plus the bf16 build's projector tolerance, on blocks whose r-th gap
    # fixes the subspace
    if lam[rank] <= 0 or lam[rank - 1] >= 1.05 * lam[rank]:
        ug = O.dequantize_u_fp4(codes_g, sb_g).T                 # [d, r]
        mag = np.abs(O.e2m1_value(codes_g))
        half = np.where(mag < 2.0, 0.25, np.where(mag < 4.0, 0.5, 1.0))
        err = np.sqrt(np.sum((half * np.repeat(np.exp2(sb_g.astype(float) - 127), 32,
                                                axis=1)) ** 2))
        po = u_o @ u_o.T
        bound = err * (2.0 * np.linalg.norm(u_o, 2) + err) + PROJ_RTOL * np.linalg.norm(po)
        assert np.linalg.norm(ug @ ug.T - po) <= bound
        stats["factors"] += 1
    for j in range(rank):
        ok_hi = j == 0 or lam[j - 1] >= GAP_COLUMN * lam[j]
        ok_lo = lam[j + 1] <= 0 or lam[j] >= GAP_COLUMN * lam[j + 1]
        if not (ok_hi and ok_lo and lam[j] > 1e-6 * lam[0]):
            continue
        stats["columns"] += 1
        col_g = O.dequantize_u_fp4(codes_g[j][None], sb_g[j][None])[0]
        sign = 1.0 if col_g @ u_o[:, j] >= 0 else -1.0   # a near-tied largest component
        cg = codes_g[j] if sign > 0 else np.where(codes_g[j] != 0, codes_g[j] ^ 8, 0)
        for g in range(d // 32):
            seg = u_o[32 * g:32 * (g + 1), j]
            amax = float(np.max(np.abs(seg)))
            e_o = O.fp4_scale_exponent(amax)
            e_g = int(sb_g[j, g]) - 127
            if e_o is None:                        # a group of zeros
                assert sb_g[j, g] == 0 and not np.any(cg[32 * g:32 * (g + 1)])
                continue
            if e_g != e_o:
                # only a group maximum within NEAR of the fitting bound 6 * 2^e
                stats["scale_boundary"] += 1
                assert abs(amax / 2.0 ** min(e_g, e_o) - 6.0) <= 6.0 * NEAR, (j, g, e_g, e_o)
                continue
            x = seg / 2.0 ** e_o
            co, cgg = codes_o[j, 32 * g:32 * (g + 1)], cg[32 * g:32 * (g + 1)]
            for t in np.nonzero(co != cgg)[0]:
                stats["code_boundary"] += 1
                vo, vg = O.e2m1_value(co[t]), O.e2m1_value(cgg[t])
                mid = 0.5 * (vo + vg)
                # neighbours across the boundary the oracle's value sits on
                assert abs(abs(x[t]) - abs(mid)) <= NEAR or abs(x[t]) <= 0.25 + NEAR, \
                    (j, g, t, x[t], vo, vg)
                grid = np.array(O.E2M1_MAGNITUDES)
                assert abs(np.searchsorted(grid, abs(vo)) - np.searchsorted(grid, abs(vg))) <= 1
            stats["codes"] += 32


def test_stats_build_fp4(fp):
    p, w = fp, fp.w
    p.build_stats()
    p.build_stats4()
    torch.cuda.synchronize()
    st16 = from_dev_bits(p.stats)
    st4 = p.stats4.cpu().numpy()
    nfull = w.seq_len // w.block
    stats = dict(columns=0, codes=0, code_boundary=0, scale_boundary=0, factors=0)
    for b in range(w.batch):
        for h in range(w.kv_heads):
            mu_g, codes_g, sb_g, pad_g = unpack_fp4_records(st4[b, h, :nfull], w.head_dim,
                                                            w.rank)
            # mu: the same bf16 values as the bf16 record's row 0
            np.testing.assert_array_equal(mu_g, bits_to_f64(st16[b, h, :nfull, 0]))
            keys = p.keys(b, h)
            for j in range(nfull):
                check_fp4_block(mu_g[j], codes_g[j], sb_g[j], pad_g[j],
                                keys[j * w.block:(j + 1) * w.block], w.rank, stats)
    # untouched past the built range
    assert np.all(st4[:, :, nfull:] == 0)
    print(f"fp4 stats: {stats}")
    assert stats["factors"] > 0
    assert stats["code_boundary"] <= 0.01 * max(1, stats["codes"])
    assert p.device_status() == 0


def test_planted_blocks_fp4():
    """Blocks with exactly known covariance: codes and exponents equal the
    oracle's except at boundary cases."""
    w = W["single_32k"].scaled(seq_len=64 * 8, batch=1, q_heads=4, kv_heads=1, rank=6)
    p = Fp4Problem(w)
    rng = np.random.default_rng(7)
    from test_oracle_pins import planted_block
    kb = p.k_bits.copy()
    want = []
    for j in range(8):
        lam = np.sort(rng.uniform(0.2, 3.0, size=6))[::-1] * (1 + j)
        lam = lam * (1.5 ** -np.arange(6))             # well separated
        mu = 0.3 * rng.standard_normal(w.head_dim)
        keys, _ = planted_block(64, w.head_dim, lam, mu, seed=j)
        kb[0, 0, j * 64:(j + 1) * 64] = to_bf16_bits(keys)
        want.append(bits_to_f64(to_bf16_bits(keys)))
    p.k = to_dev(kb)
    p.build_stats4(0, 8)
    st4 = p.stats4.cpu().numpy()
    mu_g, codes_g, sb_g, pad_g = unpack_fp4_records(st4[0, 0, :8], w.head_dim, w.rank)
    stats = dict(columns=0, codes=0, code_boundary=0, scale_boundary=0, factors=0)
    for j in range(8):
        mu_o = O.round_to_bf16(want[j].mean(axis=0))
        np.testing.assert_array_equal(mu_g[j], mu_o)
        check_fp4_block(mu_g[j], codes_g[j], sb_g[j], pad_g[j], want[j], w.rank, stats)
    print(f"planted fp4 stats: {stats}")
    assert stats["columns"] >= 8 * 5
    assert p.device_status() == 0


def test_end_to_end_fp4(fp):
    """FP4 statistics, selection and decode against the oracle: each selection
    flip explained by the records (the GPU's FP4 records against the oracle's
    quantisation of the exact factor), outputs equal to the oracle's attention
    over the GPU's selection."""
    p, w = fp, fp.w
    p.build_stats4()
    p.select4()
    p.decode()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    out = p.out.cpu().numpy()
    raw = p.stats4.cpu().numpy()
    G = w.group
    scale = 1 / math.sqrt(w.head_dim)
    nfull = w.seq_len // w.block
    flips = 0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            orc = O.fp4_record_values(*p.oracle_records4(b, h))
            mu_g, codes_g, sb_g, _ = unpack_fp4_records(raw[b, h, :nfull], w.head_dim, w.rank)
            gpu = O.fp4_record_values(mu_g, codes_g, sb_g)
            got = idx[b, h, :n[b, h]]
            nd, _, _ = explain_selection(w, p.q_group(b, h), got, gpu, orc)
            flips += nd > 0
            o, _ = O.sparse_attention(p.q_group(b, h), p.keys(b, h), p.values(b, h),
                                      got.astype(np.int64), w.seq_len, w.block, scale)
            assert np.max(np.abs(out[b, h * G:(h + 1) * G] - o)) <= OUT_ATOL
    print(f"fp4 end-to-end selections differing from the oracle's: {flips} of "
          f"{w.batch * w.kv_heads} pairs (each explained by its records)")
    assert p.device_status() == 0


def test_fp4_needles_are_found():
    """The needle blocks planted for the group's queries are selected from FP4
    records as from bf16 ones."""
    w = W["batched_needles_32k"].scaled(batch=2, seq_len=8192)
    p = Fp4Problem(w)
    from workloads import needle_block_list
    p.build_stats()
    p.select()
    sel16 = p.idx.cpu().numpy().copy(), p.n_sel.cpu().numpy().copy()
    p.build_stats4()
    p.select4()
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    found16 = found4 = total = 0
    for b in range(w.batch):
        for h in range(w.kv_heads):
            needles = set(needle_block_list(w, b, h))
            total += len(needles)
            found16 += len(needles & set(sel16[0][b, h, :sel16[1][b, h]].tolist()))
            found4 += len(needles & set(idx[b, h, :n[b, h]].tolist()))
    print(f"needle blocks found: bf16 {found16}/{total}, fp4 {found4}/{total}")
    assert total > 0 and found4 >= found16 - max(1, total // 50)
    assert p.device_status() == 0


@pytest.mark.parametrize("name,pairs", [
    ("batched_needles_32k", [(0, 0), (17, 3), (31, 7)]),
    ("build_256k", [(0, 0), (0, 5)]),
])
def test_select_fp4_at_full_size(name, pairs):
    """Selection over FP4 records in the launch the full workload gets: at
    batched_needles_32k every CTA streams a whole pair's 503 candidates
    (~36 passes through its record ring and both tensor-memory
    accumulators); build_256k splits 4079 candidates per pair over many CTAs
    and ranks them with the grouped top-k (more than 1024 candidates).  The
    oracle's FP4 records are uploaded for the sampled pairs (all other pairs
    keep zero records, which are valid records too)."""
    from workloads import make_kv_slice, make_queries
    w = W[name]
    dims = dict(batch=w.batch, num_q_heads=w.q_heads, num_kv_heads=w.kv_heads,
                head_dim=w.head_dim, block_size=w.block, rank=w.rank,
                capacity_tokens=w.cap, stats_format=cb.COBS_STATS_FP4)
    rec = cb.cobs_stats_record_bytes(dims)
    q_bits = make_queries(w)
    q = to_dev(q_bits)
    nb_cap = w.cap // w.block
    nfull = w.seq_len // w.block
    stats4 = torch.zeros((w.batch, w.kv_heads, nb_cap, rec), dtype=torch.uint8, device="cuda")
    nsm = cb.cobs_selected_capacity(dims, w.top_k, w.sink_blocks, w.local_tokens)
    idx = torch.full((w.batch, w.kv_heads, nsm), -7, dtype=torch.int32, device="cuda")
    n_sel = torch.zeros((w.batch, w.kv_heads), dtype=torch.int32, device="cuda")
    scores = torch.full((w.batch, w.kv_heads, nb_cap), float("nan"), device="cuda")
    ws_bytes = cb.cobs_workspace_bytes(dims, w.top_k, w.sink_blocks, w.local_tokens)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    cb.cobs_workspace_init(ws, ws_bytes)
    from harness import pack_fp4_records
    parts = {}
    for (b, h) in pairs:
        kb, _ = make_kv_slice(w, b, h, q_bits if w.needles else None)
        parts[(b, h)] = O.build_block_records_fp4(bits_to_f64(kb), w.block, w.rank, 0, nfull)
        stats4[b, h, :nfull] = torch.from_numpy(pack_fp4_records(*parts[(b, h)])).cuda()
    cb.cobs_select_blocks(dims, q, stats4, w.seq_len, w.top_k, w.sink_blocks,
                          w.local_tokens, idx, nsm, n_sel, scores, ws, ws_bytes)
    idx_h, n_h, sc_h = idx.cpu().numpy(), n_sel.cpu().numpy(), scores.cpu().numpy()
    G = w.group
    _, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
    for (b, h), pr in parts.items():
        qg = bits_to_f64(q_bits[b, h * G:(h + 1) * G])
        sel, s = O.select_from_records(qg, O.fp4_record_values(*pr), w.seq_len, w.block,
                                       w.top_k, w.sink_blocks, w.local_tokens)
        got = idx_h[b, h, :n_h[b, h]]
        assert len(got) == len(sel) and np.all(np.diff(got) > 0)
        assert selection_mismatch(got, sel, s, w) == [], (b, h)
        np.testing.assert_allclose(sc_h[b, h, c0:c1], s[c0:c1], rtol=0,
                                   atol=TIE_RTOL * max(1, np.max(np.abs(s))))
    assert cb.cobs_read_device_status(ws, ws_bytes) == 0


def test_select_fp4_misaligned_stats_uses_widening_kernel():
    """FP4 records 16-byte but not 32-byte aligned: the tensor-core kernel's
    code map needs 32-byte alignment, so the selection falls back to the
    kernel that widens the codes in shared memory, and still equals the
    oracle's selection from the records (ties reported)."""
    w = CASES["needles_b2_r8"]
    p = Fp4Problem(w, poison="nan")
    orc = {}
    for b in range(w.batch):
        for h in range(w.kv_heads):
            parts = p.oracle_records4(b, h)
            p.upload_records4(b, h, parts)
            orc[(b, h)] = oracle_selection4(p, b, h, parts)
    # the same records, starting 16 bytes past a 32-byte boundary
    flat = torch.zeros(p.stats4.numel() + 64, dtype=torch.uint8, device="cuda")
    off = (16 - flat.data_ptr() % 32) % 32
    shifted = flat[off:off + p.stats4.numel()].view(p.stats4.shape)
    shifted.copy_(p.stats4)
    assert shifted.data_ptr() % 32 == 16
    cb.cobs_select_blocks(p.dims4, p.q, shifted, w.seq_len, w.top_k, w.sink_blocks,
                          w.local_tokens, p.idx, p.idx.shape[-1], p.n_sel, p.scores, p.ws,
                          p.ws_bytes)
    idx, n = p.idx.cpu().numpy(), p.n_sel.cpu().numpy()
    scores = p.scores.cpu().numpy()
    _, c0, c1 = O.block_partition(w.seq_len, w.block, w.sink_blocks, w.local_tokens)
    for (b, h), (sel, s) in orc.items():
        got = idx[b, h, :n[b, h]]
        assert np.all(np.diff(got) > 0)
        assert n[b, h] == len(sel)
        assert selection_mismatch(got, sel, s, w) == [], (b, h)
        np.testing.assert_allclose(scores[b, h, c0:c1], s[c0:c1],
                                   rtol=0, atol=TIE_RTOL * max(1, np.max(np.abs(s))))
    assert p.device_status() == 0
