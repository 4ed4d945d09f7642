"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, sizes its workspace as documented, and rejects bad arguments before
touching the GPU (no compute call is made here, so these run without one)."""

import ctypes
import os
import re

import pytest

import block_sparse_long_cobs_b200 as cb
from workloads import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "cobs.h")


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"COBS_API\s+[\w\s\*]+?\b(cobs_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert len(names) == 19, names
    raw = ctypes.CDLL(cb.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    for n in names:
        assert callable(getattr(cb, n)), n


def test_version_and_status_strings():
    assert cb.cobs_abi_version() == 4
    assert cb.cobs_status_string(0) == "COBS_OK"
    assert cb.cobs_status_string(5) == "COBS_ERR_TIMEOUT"
    assert cb.cobs_status_string(99) == "COBS_ERR_UNKNOWN"


def dims_of(w, **kw):
    d = dict(batch=w.batch, num_q_heads=w.q_heads, num_kv_heads=w.kv_heads,
             head_dim=w.head_dim, block_size=w.block, rank=w.rank,
             capacity_tokens=w.cap)
    d.update(kw)
    return d


def ceil_div(a, b):
    return -(-a // b)


def align(x):
    return (x + 255) // 256 * 256


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_selected_capacity_and_workspace_size(name):
    w = WORKLOADS[name]
    d = dims_of(w)
    nsm = cb.cobs_selected_capacity(d, w.top_k, w.sink_blocks, w.local_tokens)
    assert nsm == min(w.cap // 64, w.top_k + w.sink_blocks + ceil_div(w.local_tokens, 64) + 1)
    ws = cb.cobs_workspace_bytes(d, w.top_k, w.sink_blocks, w.local_tokens)
    pairs = w.batch * w.kv_heads
    # status, selection tickets, decode tickets + the decode work counters (2),
    # the hand-off (epoch, count, ready list), scores, split partials
    want = 256 + align(pairs * 4) + align((pairs + 2) * 4) + align(16 + pairs * 8) + \
        align(pairs * (w.cap // 64) * 4) + align(w.batch * w.q_heads * nsm * (w.head_dim + 2) * 4)
    assert ws == want


@pytest.mark.parametrize("kw,code", [
    (dict(num_q_heads=12, num_kv_heads=4), cb.COBS_ERR_UNSUPPORTED),   # G = 3
    (dict(num_q_heads=10, num_kv_heads=4), cb.COBS_ERR_INVALID_ARG),
    (dict(head_dim=96), cb.COBS_ERR_UNSUPPORTED),
    (dict(block_size=32), cb.COBS_ERR_UNSUPPORTED),
    (dict(rank=17), cb.COBS_ERR_UNSUPPORTED),
    (dict(rank=-1), cb.COBS_ERR_UNSUPPORTED),
    (dict(capacity_tokens=1000), cb.COBS_ERR_INVALID_ARG),
    (dict(batch=0), cb.COBS_ERR_INVALID_ARG),
])
def test_bad_dims_rejected_everywhere(kw, code):
    w = WORKLOADS["single_32k"]
    d = dims_of(w, **kw)
    fake = 1 << 20                     # never dereferenced: rejected first
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_build_block_stats(d, fake, 0, 1, fake, fake, 1 << 20)
    assert e.value.status == code
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_select_blocks(d, fake, fake, 100, 8, 1, 64, fake, 64, fake, None, fake, 1 << 20)
    assert e.value.status == code
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_sparse_decode(d, fake, fake, fake, fake, fake, 10, 100, 0.1, fake, fake,
                              fake, 1 << 20)
    assert e.value.status == code
    assert cb.cobs_selected_capacity is not None
    assert cb.lib.cobs_workspace_bytes(ctypes.byref(cb.cobs_dims(**d)), 8, 1, 64) == 0
    assert len(cb.cobs_last_error()) > 0


def test_pointer_and_range_checks():
    w = WORKLOADS["single_32k"]
    d = dims_of(w)
    A = 1 << 20
    ws_need = cb.cobs_workspace_bytes(d, w.top_k, 1, w.local_tokens)
    nsm = cb.cobs_selected_capacity(d, w.top_k, 1, w.local_tokens)
    cases = [
        # build: null, misaligned, block range, workspace
        (lambda: cb.cobs_build_block_stats(d, None, 0, 1, A, A, 4096), cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_build_block_stats(d, A + 8, 0, 1, A, A, 4096), cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_build_block_stats(d, A, 0, w.cap // 64 + 1, A, A, 4096),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_build_block_stats(d, A, 5, 4, A, A, 4096), cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_build_block_stats(d, A, -1, 4, A, A, 4096), cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_build_block_stats(d, A, 0, 4, A, None, 4096), cb.COBS_ERR_WORKSPACE),
        (lambda: cb.cobs_build_block_stats(d, A, 0, 4, A, A, 16), cb.COBS_ERR_WORKSPACE),
        # select
        (lambda: cb.cobs_select_blocks(d, A, A, 0, 8, 1, 64, A, 64, A, None, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_select_blocks(d, A, A, w.cap + 1, 8, 1, 64, A, 64, A, None, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_select_blocks(d, A, A, 100, -1, 1, 64, A, 64, A, None, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_select_blocks(d, A, A, 100, 8, 1, 64, None, 64, A, None, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_select_blocks(d, A, A, 100, 8, 1, 64, A, 64, A + 4, None, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_select_blocks(d, A, A, 100, 8, 1, 64, A, 64, A, A + 2, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_select_blocks(d, A, A, 100, 16, 1, 512, A, 64, A, None, A, 1024),
         cb.COBS_ERR_WORKSPACE),
        (lambda: cb.cobs_select_blocks(d, A, A, 100, 16, 1, 512, A, 25, A, None, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),                       # idx row too short for 26 blocks
        # decode
        (lambda: cb.cobs_sparse_decode(d, A, A, A, A, A, 0, 100, 0.1, A, A, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_sparse_decode(d, A, A, A, A, A, nsm, 100, 0.0, A, A, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_sparse_decode(d, A, A, A, A, A, nsm, 100, float("nan"), A, A, A,
                                       ws_need), cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_sparse_decode(d, A, A, A, A, A, nsm + 1, 100, 0.1, A, A, A, ws_need),
         cb.COBS_ERR_WORKSPACE),
        (lambda: cb.cobs_sparse_decode(d, A, A, None, A, A, nsm, 100, 0.1, A, A, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_sparse_decode(d, A, A, A, A, A, nsm, 100, 0.1, A, A + 12, A, ws_need),
         cb.COBS_ERR_INVALID_ARG),
        # workspace helpers
        (lambda: cb.cobs_workspace_init(None, 4096), cb.COBS_ERR_WORKSPACE),
        (lambda: cb.cobs_workspace_init(A + 1, 4096), cb.COBS_ERR_INVALID_ARG),
        (lambda: cb.cobs_read_device_status(None, 4096), cb.COBS_ERR_WORKSPACE),
    ]
    for fn, code in cases:
        with pytest.raises(cb.CobsError) as e:
            fn()
        assert e.value.status == code, (e.value, code)


def test_status_read_rejects_null_output():
    st = cb.lib.cobs_read_device_status(ctypes.c_void_p(1 << 20), 4096, None, None)
    assert st == cb.COBS_ERR_INVALID_ARG


def test_selection_limits_are_checked_on_the_host():
    """top_k above 4096, and settings whose exact top-k survivors could
    overflow the selection kernel's shared memory, are refused before launch."""
    A = 1 << 20
    w = WORKLOADS["single_32k"]
    d = dims_of(w)
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_select_blocks(d, A, A, 100, 4097, 1, 64, A, 8192, A, None, A, 1 << 30)
    assert e.value.status == cb.COBS_ERR_UNSUPPORTED
    # head_dim 64 (a 48 KB record ring), a million-token cache, top_k 4000:
    # the candidates above the grouped bound would need ~512 KB
    d64 = dims_of(WORKLOADS["tiny_4k"], capacity_tokens=1 << 20)
    nsm = cb.cobs_selected_capacity(d64, 4000, 1, 0)
    ws = cb.cobs_workspace_bytes(d64, 4000, 1, 0)
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_select_blocks(d64, A, A, 1 << 20, 4000, 1, 0, A, nsm, A, None, A, ws)
    assert e.value.status == cb.COBS_ERR_UNSUPPORTED
    assert "shared memory" in cb.cobs_last_error()


def test_varlen_host_checks():
    A = 1 << 20
    w = WORKLOADS["single_32k"]
    d = dims_of(w)
    ws = cb.cobs_workspace_bytes(d, w.top_k, 1, w.local_tokens)
    nsm = cb.cobs_selected_capacity(d, w.top_k, 1, w.local_tokens)
    sel = lambda lens, mx: cb.cobs_select_blocks_varlen(d, A, A, lens, mx, w.top_k, 1,
                                                        w.local_tokens, A, nsm, A, None, A, ws)
    dec = lambda lens, mx: cb.cobs_sparse_decode_varlen(d, A, A, A, A, A, nsm, lens, mx, 0.1,
                                                        A, A, A, ws)
    for call in (sel, dec):
        for lens, mx, code in [(None, 100, cb.COBS_ERR_INVALID_ARG),
                               (A + 8, 100, cb.COBS_ERR_INVALID_ARG),
                               (A, 0, cb.COBS_ERR_INVALID_ARG),
                               (A, w.cap + 1, cb.COBS_ERR_INVALID_ARG)]:
            with pytest.raises(cb.CobsError) as e:
                call(lens, mx)
            assert e.value.status == code


def test_paged_host_checks():
    """Block-table arguments are checked before launch: the table itself, its
    row length against the blocks addressed, the pool size and the index
    ranges that must fit 32 bits."""
    A = 1 << 20
    w = WORKLOADS["single_32k"]
    d = dims_of(w)
    ws = cb.cobs_workspace_bytes(d, w.top_k, 1, w.local_tokens)
    nsm = cb.cobs_selected_capacity(d, w.top_k, 1, w.local_tokens)
    nb = w.cap // 64
    stats = lambda tbl, stride, pages, end: cb.cobs_build_block_stats_paged(
        d, A, pages, tbl, stride, 0, end, A, A, 4096)
    dec = lambda tbl, stride, pages, mx: cb.cobs_sparse_decode_paged(
        d, A, A, A, pages, tbl, stride, A, A, nsm, None, mx, 0.1, A, A, A, ws)
    cases = [
        (lambda: stats(None, nb, 100, 4), cb.COBS_ERR_INVALID_ARG),
        (lambda: stats(A + 4, nb, 100, 4), cb.COBS_ERR_INVALID_ARG),
        (lambda: stats(A, 3, 100, 4), cb.COBS_ERR_INVALID_ARG),        # row shorter than end
        (lambda: stats(A, nb, 0, 4), cb.COBS_ERR_INVALID_ARG),
        (lambda: stats(A, nb, 1 << 30, 4), cb.COBS_ERR_UNSUPPORTED),  # pool rows >= 2^31
        (lambda: cb.cobs_build_block_stats_paged(dims_of(w, batch=2), A, 100, A, 1 << 30, 0,
                                                 4, A, A, 4096),
         cb.COBS_ERR_UNSUPPORTED),                                      # batch x stride
        (lambda: stats(A, nb, 100, nb + 1), cb.COBS_ERR_INVALID_ARG),  # past the capacity
        (lambda: dec(None, nb, 100, 4096), cb.COBS_ERR_INVALID_ARG),
        (lambda: dec(A, 63, 100, 4096), cb.COBS_ERR_INVALID_ARG),      # needs 64 blocks
        (lambda: dec(A, 64, 0, 4096), cb.COBS_ERR_INVALID_ARG),
        (lambda: dec(A, 64, 1 << 30, 4096), cb.COBS_ERR_UNSUPPORTED),
        (lambda: dec(A, 64, 100, w.cap + 1), cb.COBS_ERR_INVALID_ARG),
    ]
    for fn, code in cases:
        with pytest.raises(cb.CobsError) as e:
            fn()
        assert e.value.status == code, (e.value, code)


def test_stats_record_bytes_and_format_checks():
    from harness import fp4_record_bytes
    for name in ("tiny_4k", "single_32k", "build_256k"):
        w = WORKLOADS[name]
        d = dims_of(w)
        assert cb.cobs_stats_record_bytes(d) == (1 + w.rank) * w.head_dim * 2
        d4 = dims_of(w, stats_format=cb.COBS_STATS_FP4)
        n = cb.cobs_stats_record_bytes(d4)
        assert n == fp4_record_bytes(w.head_dim, w.rank) and n % 16 == 0
        assert n >= 2 * w.head_dim + w.rank * w.head_dim // 2 + w.rank * w.head_dim // 32
    # d 128, r 8: 256 B of mu, 512 B of codes, 32 scale bytes
    assert cb.cobs_stats_record_bytes(dims_of(WORKLOADS["single_32k"], rank=8,
                                              stats_format=1)) == 800
    # min/max box records: lo and hi, d bf16 each, whatever the rank
    for r in (0, 8, 16):
        assert cb.cobs_stats_record_bytes(dims_of(WORKLOADS["single_32k"], rank=r,
                                                  stats_format=cb.COBS_STATS_BOX)) == 512
    assert cb.cobs_stats_record_bytes(dims_of(WORKLOADS["tiny_4k"],
                                              stats_format=cb.COBS_STATS_BOX)) == 256
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_stats_record_bytes(dims_of(WORKLOADS["single_32k"], stats_format=3))
    assert e.value.status == cb.COBS_ERR_INVALID_ARG
    with pytest.raises(cb.CobsError):
        cb.cobs_stats_record_bytes(dims_of(WORKLOADS["single_32k"], rank=0, stats_format=1))
    assert "rank" in cb.cobs_last_error()
    A = 1 << 20
    with pytest.raises(cb.CobsError) as e:   # FP4 records need a factor
        cb.cobs_build_block_stats(dims_of(WORKLOADS["single_32k"], rank=0, stats_format=1),
                                  A, 0, 1, A, A, 4096)
    assert e.value.status == cb.COBS_ERR_UNSUPPORTED
    # every call checks the format before launching anything
    A = 1 << 20
    bad = dims_of(WORKLOADS["single_32k"], stats_format=7)
    with pytest.raises(cb.CobsError) as e:
        cb.cobs_build_block_stats(bad, A, 0, 1, A, A, 4096)
    assert e.value.status == cb.COBS_ERR_INVALID_ARG


def test_fp4_record_packing_round_trip():
    """The test-side packing of oracle FP4 records follows the header's layout."""
    import numpy as np
    import oracle.cobs_oracle as O
    from harness import pack_fp4_records, unpack_fp4_records
    rng = np.random.default_rng(0)
    for d, r in ((128, 8), (64, 4), (128, 1), (64, 16)):
        keys = O.round_to_bf16(rng.normal(0, 0.5, size=(3 * 64, d)))
        mu, codes, sb = O.build_block_records_fp4(keys, 64, r, 0, 3)
        raw = pack_fp4_records(mu, codes, sb)
        m2, c2, s2, pad = unpack_fp4_records(raw, d, r)
        np.testing.assert_array_equal(m2, mu)
        np.testing.assert_array_equal(c2, codes)
        np.testing.assert_array_equal(s2, sb)
        assert raw.shape[1] % 16 == 0 and np.all(pad == 0)
        # component 1 of column 0 is the high nibble of byte 2d
        assert raw[0, 2 * d] >> 4 == codes[0, 0, 1] and raw[0, 2 * d] & 15 == codes[0, 0, 0]


def test_binding_rejects_host_and_strided_tensors():
    """Every pointer of the ABI is a device pointer: host or strided torch
    tensors are refused before the library is called."""
    import torch
    w = WORKLOADS["tiny_4k"]
    d = dims_of(w)
    host = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(TypeError):
        cb.cobs_workspace_init(host, 16)
    strided = torch.zeros((4, 8))[:, ::2]
    assert not strided.is_contiguous()
    with pytest.raises(TypeError):
        cb.cobs_build_block_stats(d, strided, 0, 1, 1 << 20, 1 << 20, 4096)


def test_subspace_dims_checks():
    """Subspace records (COBS_STATS_SUBSPACE): record size 2 d + 2 r s8 bytes
    (s8 = s rounded up to 8); s in [1, d], an aligned basis and rank >= 1 are
    required, checked before anything is launched."""
    w = WORKLOADS["single_32k"]
    A = 1 << 20
    base = dims_of(w, stats_format=cb.COBS_STATS_SUBSPACE, subspace_basis=A)
    for s, want in ((85, 256 + 2 * 8 * 88), (64, 256 + 2 * 8 * 64), (1, 256 + 2 * 8 * 8),
                    (128, 9 * 256)):
        assert cb.cobs_stats_record_bytes(dict(base, subspace_dim=s)) == want
    assert cb.cobs_stats_record_bytes(dims_of(WORKLOADS["tiny_4k"], rank=4, subspace_dim=40,
                                              stats_format=cb.COBS_STATS_SUBSPACE,
                                              subspace_basis=A)) == 128 + 2 * 4 * 40
    for bad, code in ((dict(subspace_dim=0), cb.COBS_ERR_INVALID_ARG),
                      (dict(subspace_dim=129), cb.COBS_ERR_INVALID_ARG),
                      (dict(subspace_dim=85, subspace_basis=None), cb.COBS_ERR_INVALID_ARG),
                      (dict(subspace_dim=85, subspace_basis=A + 4), cb.COBS_ERR_INVALID_ARG),
                      (dict(subspace_dim=85, rank=0), cb.COBS_ERR_UNSUPPORTED)):
        d = dict(base, **bad)
        with pytest.raises(cb.CobsError):        # a size query only says "invalid"
            cb.cobs_stats_record_bytes(d)
        with pytest.raises(cb.CobsError) as e:
            cb.cobs_build_block_stats(d, A, 0, 1, A, A, 4096)
        assert e.value.status == code, bad
    # the other formats ignore the subspace fields
    assert cb.cobs_stats_record_bytes(dims_of(w, subspace_dim=999)) == 9 * 256


def test_wait_limit_knob():
    assert cb.cobs_set_wait_limit_ns(5_000_000) == cb.COBS_OK
    assert cb.cobs_set_wait_limit_ns(0) == cb.COBS_OK     # back to the default


def test_select_and_decode_checks_both_calls_before_launching():
    """The fused call refuses anything either call would refuse, before it
    launches anything: a selection argument (top_k above 4096, idx_stride
    too short), a decode argument (softmax_scale), the workspace size."""
    A = 1 << 20
    w = WORKLOADS["single_32k"]
    d = dims_of(w)
    ws = cb.cobs_workspace_bytes(d, w.top_k, 1, w.local_tokens)
    nsm = cb.cobs_selected_capacity(d, w.top_k, 1, w.local_tokens)
    call = lambda top_k=w.top_k, stride=nsm, scale=0.1, ws_bytes=ws: cb.cobs_select_and_decode(
        d, A, A, A, A, w.seq_len, top_k, 1, w.local_tokens, scale, A, stride, A, None, A, A,
        A, ws_bytes)
    for kw, code, text in [(dict(top_k=4097), cb.COBS_ERR_UNSUPPORTED, "top_k"),
                           (dict(stride=nsm - 1), cb.COBS_ERR_INVALID_ARG, "idx_stride"),
                           (dict(scale=-1.0), cb.COBS_ERR_INVALID_ARG, "softmax_scale"),
                           (dict(scale=float("nan")), cb.COBS_ERR_INVALID_ARG, "softmax_scale"),
                           (dict(ws_bytes=ws - 256), cb.COBS_ERR_WORKSPACE, "workspace")]:
        with pytest.raises(cb.CobsError) as e:
            call(**kw)
        assert e.value.status == code, kw
        assert text in cb.cobs_last_error(), (kw, cb.cobs_last_error())
