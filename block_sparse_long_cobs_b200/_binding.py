"""Thin Python binding of the COBS block-sparse decode C ABI (``include/cobs.h``).

Argument marshalling only: every function here forwards to the function of
the same name in ``libcobs_b200.so`` (built in-tree by
``python -m block_sparse_long_cobs_b200.build``); all computation happens in
the library's CUDA kernels.  Tensors may be given as torch tensors (their
``data_ptr()`` is passed), integer addresses or ``None`` (NULL).  Streams may
be a ``torch.cuda.Stream``, an integer handle or ``None`` (legacy default
stream).  Importing this module fails if the library has not been built: there
is no fallback path.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "CobsError", "cobs_dims", "LIB_PATH", "lib",
    "cobs_abi_version", "cobs_stats_record_bytes", "cobs_selected_capacity",
    "cobs_workspace_bytes", "COBS_STATS_BF16", "COBS_STATS_FP4", "COBS_STATS_BOX",
    "COBS_STATS_SUBSPACE",
    "cobs_workspace_init", "cobs_build_block_stats", "cobs_select_blocks",
    "cobs_sparse_decode", "cobs_sparse_decode_no_alloc", "cobs_select_blocks_varlen",
    "cobs_sparse_decode_varlen", "cobs_build_block_stats_paged", "cobs_sparse_decode_paged",
    "cobs_select_and_decode", "cobs_read_device_status", "cobs_no_alloc_read_status",
    "cobs_set_wait_limit_ns",
    "cobs_last_error",
    "cobs_status_string",
    "COBS_OK", "COBS_ERR_INVALID_ARG", "COBS_ERR_UNSUPPORTED",
    "COBS_ERR_WORKSPACE", "COBS_ERR_CUDA", "COBS_ERR_TIMEOUT", "COBS_ERR_DEVICE",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libcobs_b200.so")

COBS_OK = 0
COBS_ERR_INVALID_ARG = 1
COBS_ERR_UNSUPPORTED = 2
COBS_ERR_WORKSPACE = 3
COBS_ERR_CUDA = 4
COBS_ERR_TIMEOUT = 5
COBS_ERR_DEVICE = 6

COBS_STATS_BF16 = 0     # block records: mu and U in bf16
COBS_STATS_FP4 = 1      # block records: mu in bf16, U in scaled FP4 (E2M1)
COBS_STATS_BOX = 2      # block records: per-dimension min and max of the keys (bf16)
COBS_STATS_SUBSPACE = 3  # block records: mu in bf16, U projected on a query subspace (bf16)


class CobsError(RuntimeError):
    """A COBS call returned a non-OK status."""

    def __init__(self, func: str, status: int, message: str):
        super().__init__(f"{func}: {cobs_status_string(status)}: {message}")
        self.status = status


class cobs_dims(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("num_q_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("rank", ctypes.c_int32),
        ("capacity_tokens", ctypes.c_int64),
        ("stats_format", ctypes.c_int32),       # COBS_STATS_BF16 / _FP4 / _BOX / _SUBSPACE
        ("subspace_dim", ctypes.c_int32),       # s of COBS_STATS_SUBSPACE records
        ("subspace_basis", ctypes.c_void_p),    # device [Hkv][s][d] fp32 basis
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"COBS CUDA library not found at {LIB_PATH}; build it with "
            "`python -m block_sparse_long_cobs_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ, F32 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                            ctypes.c_size_t, ctypes.c_float)
    D = ctypes.POINTER(cobs_dims)
    sig = {
        "cobs_abi_version": (I32, []),
        "cobs_stats_record_bytes": (I64, [D]),
        "cobs_selected_capacity": (I32, [D, I32, I32, I32]),
        "cobs_workspace_bytes": (SZ, [D, I32, I32, I32]),
        "cobs_workspace_init": (I32, [P, SZ, P]),
        "cobs_build_block_stats": (I32, [D, P, I64, I64, P, P, SZ, P]),
        "cobs_select_blocks": (I32, [D, P, P, I64, I32, I32, I32, P, I32, P, P, P, SZ, P]),
        "cobs_sparse_decode": (I32, [D, P, P, P, P, P, I32, I64, F32, P, P, P, SZ, P]),
        "cobs_sparse_decode_no_alloc": (I32, [D, P, P, P, P, P, I32, I64, F32, P, P, P]),
        "cobs_select_blocks_varlen": (I32, [D, P, P, P, I64, I32, I32, I32, P, I32, P, P, P,
                                            SZ, P]),
        "cobs_sparse_decode_varlen": (I32, [D, P, P, P, P, P, I32, P, I64, F32, P, P, P, SZ, P]),
        "cobs_build_block_stats_paged": (I32, [D, P, I64, P, I32, I64, I64, P, P, SZ, P]),
        "cobs_sparse_decode_paged": (I32, [D, P, P, P, I64, P, I32, P, P, I32, P, I64, F32, P,
                                           P, P, SZ, P]),
        "cobs_select_and_decode": (I32, [D, P, P, P, P, I64, I32, I32, I32, F32, P, I32, P, P,
                                         P, P, P, SZ, P]),
        "cobs_read_device_status": (I32, [P, SZ, ctypes.POINTER(I32), P]),
        "cobs_no_alloc_read_status": (I32, [ctypes.POINTER(I32), P]),
        "cobs_set_wait_limit_ns": (I32, [ctypes.c_uint64]),
        "cobs_last_error": (ctypes.c_char_p, []),
        "cobs_status_string": (ctypes.c_char_p, [I32]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def _ptr(x):
    """Device address of a buffer argument (every pointer of the C ABI is a
    device pointer): an int is taken as is; a torch tensor must be a
    contiguous CUDA tensor (a host or strided tensor would hand the kernels a
    wrong address)."""
    if x is None:
        return None
    if isinstance(x, int):
        return ctypes.c_void_p(x)
    if hasattr(x, "data_ptr"):
        if hasattr(x, "is_cuda") and not x.is_cuda:
            raise TypeError("tensor arguments must be CUDA tensors (got a host tensor)")
        if hasattr(x, "is_contiguous") and not x.is_contiguous():
            raise TypeError("tensor arguments must be contiguous")
        return ctypes.c_void_p(x.data_ptr())
    if hasattr(x, "ctypes"):
        return ctypes.c_void_p(x.ctypes.data)
    raise TypeError(f"cannot pass {type(x).__name__} as a pointer")


def _stream(s):
    if s is None:
        return None
    if isinstance(s, int):
        return ctypes.c_void_p(s)
    return ctypes.c_void_p(s.cuda_stream)


def _check(func: str, status: int, check: bool) -> int:
    if check and status != COBS_OK:
        raise CobsError(func, status, cobs_last_error())
    return status


def _dims(d) -> cobs_dims:
    if isinstance(d, cobs_dims):
        return d
    d = dict(d)
    if d.get("subspace_basis") is not None:
        d["subspace_basis"] = _ptr(d["subspace_basis"]).value
    return cobs_dims(**d)


def cobs_abi_version() -> int:
    return lib.cobs_abi_version()


def cobs_stats_record_bytes(dims) -> int:
    """Bytes of one block record for dims' stats_format."""
    n = lib.cobs_stats_record_bytes(ctypes.byref(_dims(dims)))
    if n <= 0:
        raise CobsError("cobs_stats_record_bytes", COBS_ERR_INVALID_ARG, cobs_last_error())
    return n


def cobs_last_error() -> str:
    return lib.cobs_last_error().decode()


def cobs_status_string(status: int) -> str:
    return lib.cobs_status_string(status).decode()


def cobs_selected_capacity(dims, top_k, sink_blocks, local_tokens) -> int:
    n = lib.cobs_selected_capacity(ctypes.byref(_dims(dims)), top_k, sink_blocks,
                                   local_tokens)
    if n < 0:
        raise CobsError("cobs_selected_capacity", COBS_ERR_INVALID_ARG, cobs_last_error())
    return n


def cobs_workspace_bytes(dims, top_k, sink_blocks, local_tokens) -> int:
    n = lib.cobs_workspace_bytes(ctypes.byref(_dims(dims)), top_k, sink_blocks,
                                 local_tokens)
    if n == 0:
        raise CobsError("cobs_workspace_bytes", COBS_ERR_INVALID_ARG, cobs_last_error())
    return n


def cobs_workspace_init(ws, ws_bytes, stream=None, check=True) -> int:
    return _check("cobs_workspace_init",
                  lib.cobs_workspace_init(_ptr(ws), ws_bytes, _stream(stream)), check)


def cobs_build_block_stats(dims, k, block_begin, block_end, stats, ws, ws_bytes,
                           stream=None, check=True) -> int:
    st = lib.cobs_build_block_stats(ctypes.byref(_dims(dims)), _ptr(k), block_begin,
                                    block_end, _ptr(stats), _ptr(ws), ws_bytes,
                                    _stream(stream))
    return _check("cobs_build_block_stats", st, check)


def cobs_select_blocks(dims, q, stats, seq_len, top_k, sink_blocks, local_tokens,
                       idx, idx_stride, n_sel, scores_opt, ws, ws_bytes, stream=None,
                       check=True) -> int:
    st = lib.cobs_select_blocks(ctypes.byref(_dims(dims)), _ptr(q), _ptr(stats), seq_len,
                                top_k, sink_blocks, local_tokens, _ptr(idx), idx_stride,
                                _ptr(n_sel), _ptr(scores_opt), _ptr(ws), ws_bytes,
                                _stream(stream))
    return _check("cobs_select_blocks", st, check)


def cobs_sparse_decode(dims, q, k, v, idx, n_sel, idx_stride, seq_len, softmax_scale,
                       out, lse, ws, ws_bytes, stream=None, check=True) -> int:
    st = lib.cobs_sparse_decode(ctypes.byref(_dims(dims)), _ptr(q), _ptr(k), _ptr(v),
                                _ptr(idx), _ptr(n_sel), idx_stride, seq_len,
                                ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
                                _ptr(ws), ws_bytes, _stream(stream))
    return _check("cobs_sparse_decode", st, check)


def cobs_select_and_decode(dims, q, stats, k, v, seq_len, top_k, sink_blocks, local_tokens,
                           softmax_scale, idx, idx_stride, n_sel, scores_opt, out, lse, ws,
                           ws_bytes, stream=None, check=True) -> int:
    st = lib.cobs_select_and_decode(ctypes.byref(_dims(dims)), _ptr(q), _ptr(stats), _ptr(k),
                                    _ptr(v), seq_len, top_k, sink_blocks, local_tokens,
                                    ctypes.c_float(softmax_scale), _ptr(idx), idx_stride,
                                    _ptr(n_sel), _ptr(scores_opt), _ptr(out), _ptr(lse),
                                    _ptr(ws), ws_bytes, _stream(stream))
    return _check("cobs_select_and_decode", st, check)


def cobs_sparse_decode_no_alloc(dims, q, k, v, idx, n_sel, idx_stride, seq_len,
                                softmax_scale, out, lse, stream=None, check=True) -> int:
    """cobs_sparse_decode without a workspace: for callers that cannot give the
    library device memory; it uses the library's own fixed 16 MiB array."""
    st = lib.cobs_sparse_decode_no_alloc(ctypes.byref(_dims(dims)), _ptr(q), _ptr(k), _ptr(v),
                                         _ptr(idx), _ptr(n_sel), idx_stride, seq_len,
                                         ctypes.c_float(softmax_scale), _ptr(out), _ptr(lse),
                                         _stream(stream))
    return _check("cobs_sparse_decode_no_alloc", st, check)


def cobs_select_blocks_varlen(dims, q, stats, seq_lens, max_seq_len, top_k, sink_blocks,
                              local_tokens, idx, idx_stride, n_sel, scores_opt, ws, ws_bytes,
                              stream=None, check=True) -> int:
    """cobs_select_blocks with per-sequence lengths (seq_lens: device int64 [batch])."""
    st = lib.cobs_select_blocks_varlen(ctypes.byref(_dims(dims)), _ptr(q), _ptr(stats),
                                       _ptr(seq_lens), max_seq_len, top_k, sink_blocks,
                                       local_tokens, _ptr(idx), idx_stride, _ptr(n_sel),
                                       _ptr(scores_opt), _ptr(ws), ws_bytes, _stream(stream))
    return _check("cobs_select_blocks_varlen", st, check)


def cobs_sparse_decode_varlen(dims, q, k, v, idx, n_sel, idx_stride, seq_lens, max_seq_len,
                              softmax_scale, out, lse, ws, ws_bytes, stream=None,
                              check=True) -> int:
    """cobs_sparse_decode with per-sequence lengths (seq_lens: device int64 [batch])."""
    st = lib.cobs_sparse_decode_varlen(ctypes.byref(_dims(dims)), _ptr(q), _ptr(k), _ptr(v),
                                       _ptr(idx), _ptr(n_sel), idx_stride, _ptr(seq_lens),
                                       max_seq_len, ctypes.c_float(softmax_scale), _ptr(out),
                                       _ptr(lse), _ptr(ws), ws_bytes, _stream(stream))
    return _check("cobs_sparse_decode_varlen", st, check)


def cobs_build_block_stats_paged(dims, k_pool, n_pages, block_table, table_stride,
                                 block_begin, block_end, stats, ws, ws_bytes, stream=None,
                                 check=True) -> int:
    """cobs_build_block_stats over a page pool [n_pages, Hkv, 64, d] addressed through
    block_table (device int32 [batch, table_stride])."""
    st = lib.cobs_build_block_stats_paged(ctypes.byref(_dims(dims)), _ptr(k_pool), n_pages,
                                          _ptr(block_table), table_stride, block_begin,
                                          block_end, _ptr(stats), _ptr(ws), ws_bytes,
                                          _stream(stream))
    return _check("cobs_build_block_stats_paged", st, check)


def cobs_sparse_decode_paged(dims, q, k_pool, v_pool, n_pages, block_table, table_stride,
                             idx, n_sel, idx_stride, seq_lens, max_seq_len, softmax_scale,
                             out, lse, ws, ws_bytes, stream=None, check=True) -> int:
    """cobs_sparse_decode over page pools; seq_lens (device int64 [batch]) or None."""
    st = lib.cobs_sparse_decode_paged(ctypes.byref(_dims(dims)), _ptr(q), _ptr(k_pool),
                                      _ptr(v_pool), n_pages, _ptr(block_table), table_stride,
                                      _ptr(idx), _ptr(n_sel), idx_stride, _ptr(seq_lens),
                                      max_seq_len, ctypes.c_float(softmax_scale), _ptr(out),
                                      _ptr(lse), _ptr(ws), ws_bytes, _stream(stream))
    return _check("cobs_sparse_decode_paged", st, check)


def cobs_read_device_status(ws, ws_bytes, stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    out = ctypes.c_int32(0)
    st = lib.cobs_read_device_status(_ptr(ws), ws_bytes, ctypes.byref(out),
                                     _stream(stream))
    _check("cobs_read_device_status", st, True)
    return out.value


def cobs_no_alloc_read_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the status word of the
    allocation-free decode's fixed array on the current device."""
    out = ctypes.c_int32(0)
    st = lib.cobs_no_alloc_read_status(ctypes.byref(out), _stream(stream))
    _check("cobs_no_alloc_read_status", st, True)
    return out.value


def cobs_set_wait_limit_ns(limit_ns: int) -> int:
    """Limit of the statistics kernel's first bounded device wait (0: the
    default 2 s); a testing and diagnostic knob."""
    return _check("cobs_set_wait_limit_ns", lib.cobs_set_wait_limit_ns(int(limit_ns)), True)
