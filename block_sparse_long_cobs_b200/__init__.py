"""COBS block-sparse attention decode for B200 (sm_100a): Python binding.

The functions (``cobs_build_block_stats``, ``cobs_select_blocks``,
``cobs_sparse_decode``, ...) forward to the C ABI of ``libcobs_b200.so``
(declared in ``include/cobs.h``); see ``_binding.py``.  The library is loaded
on first use, and that first use raises ImportError if it has not been built
(``python -m block_sparse_long_cobs_b200.build``): there is no fallback path.
"""

from importlib import import_module as _import_module

__all__ = [
    "CobsError", "cobs_dims", "LIB_PATH", "lib",
    "cobs_abi_version", "cobs_stats_record_bytes", "cobs_selected_capacity",
    "cobs_workspace_bytes", "COBS_STATS_BF16", "COBS_STATS_FP4", "COBS_STATS_BOX",
    "COBS_STATS_SUBSPACE",
    "cobs_workspace_init", "cobs_build_block_stats", "cobs_select_blocks",
    "cobs_sparse_decode", "cobs_sparse_decode_no_alloc", "cobs_select_and_decode",
    "cobs_select_blocks_varlen",
    "cobs_sparse_decode_varlen", "cobs_build_block_stats_paged", "cobs_sparse_decode_paged",
    "cobs_read_device_status", "cobs_no_alloc_read_status", "cobs_set_wait_limit_ns",
    "cobs_last_error", "cobs_status_string",
    "COBS_OK", "COBS_ERR_INVALID_ARG", "COBS_ERR_UNSUPPORTED",
    "COBS_ERR_WORKSPACE", "COBS_ERR_CUDA", "COBS_ERR_TIMEOUT", "COBS_ERR_DEVICE",
]


def __getattr__(name):
    if name in __all__:
        return getattr(_import_module("._binding", __name__), name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
