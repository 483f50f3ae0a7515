"""ctypes declarations of libpkv.so (include/pkv.h).  Loading is lazy and loud:
if the library is missing or fails to load, every call raises."""

from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpkv.so")

PKV_OK = 0
STATUS_NAMES = {0: "PKV_OK", 1: "PKV_ERR_INVALID_ARG", 2: "PKV_ERR_UNSUPPORTED",
                3: "PKV_ERR_NO_FREE_BLOCK", 4: "PKV_ERR_CUDA", 5: "PKV_ERR_WORKSPACE_TOO_SMALL"}
PKV_F16, PKV_BF16 = 0, 1

DEVERR_BAD_BLOCK_ID = 1
DEVERR_BAD_CONTEXT_LEN = 2
DEVERR_BAD_SLOT = 4
DEVERR_WAIT_TIMEOUT = 8
DEVERR_BAD_PAIR = 16
STATIC_SCRATCH_BYTES = 16 << 20

# Every function include/pkv.h declares (checked by the tests against the header).
EXPORTS = (
    "paged_kv_append", "copy_blocks", "swap_blocks", "paged_attention_workspace_bytes", "paged_attention_decode",
    "paged_attention_decode_static_scratch", "paged_attention_prefill",
    "paged_attention_decode_shared_prefix", "paged_attention_shared_prefix_workspace_bytes",
    "pkv_pool_create", "pkv_pool_destroy", "pkv_seq_new", "pkv_seq_fork", "pkv_seq_reserve",
    "pkv_seq_reserve_tokens", "pkv_seq_new_cached", "pkv_pool_reserve_batch",
    "pkv_seq_cow", "pkv_seq_free", "pkv_seq_swap_out", "pkv_seq_swap_in", "pkv_seq_len", "pkv_seq_block_table", "pkv_pool_block_tables",
    "pkv_pool_refcount", "pkv_pool_free_list", "pkv_pool_stats", "pkv_shared_prefix_groups",
    "pkv_launch_count", "pkv_last_error", "pkv_status_string", "pkv_selftest_wait_timeout",
)


class PkvError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class PoolExhausted(PkvError):
    """PKV_ERR_NO_FREE_BLOCK: the free pool cannot cover the request."""


class CacheDesc(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("dtype", ctypes.c_int)]


class Stats(ctypes.Structure):
    _fields_ = [("free_blocks", ctypes.c_int64), ("allocated_slots", ctypes.c_int64),
                ("live_slots", ctypes.c_int64), ("live_tokens", ctypes.c_int64),
                ("shared_blocks", ctypes.c_int64), ("num_seqs", ctypes.c_int64),
                ("swapped_seqs", ctypes.c_int64), ("cached_blocks", ctypes.c_int64)]


_lock = threading.Lock()
_lib = None


def load():
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libpkv.so is not built ({LIB_PATH}); run "
                                  "`python -m paged_kv_cache_360_b200._build`")
            lib = ctypes.CDLL(LIB_PATH)
            p, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
            P = ctypes.POINTER
            st = ctypes.c_int
            sig = {
                "paged_kv_append": (st, [P(CacheDesc), p, p, p, p, p, i32, p, p]),
                "copy_blocks": (st, [P(CacheDesc), p, p, p, i32, p, p]),
                "swap_blocks": (st, [P(CacheDesc), p, p, p, p, p, i32, i32, p, p]),
                "paged_attention_workspace_bytes": (sz, [P(CacheDesc), i32, i32, i32, i32]),
                "paged_attention_decode": (st, [P(CacheDesc), p, p, p, p, p, i32, p, i32, i32,
                                                ctypes.c_float, i32, p, sz, p, p]),
                "paged_attention_decode_static_scratch": (st, [P(CacheDesc), p, p, p, p, p, i32, p,
                                                               i32, i32, ctypes.c_float, i32, p, p]),
                "paged_attention_prefill": (st, [P(CacheDesc), p, p, p, p, p, i32, p, p, i32, i32,
                                                 i32, ctypes.c_float, p, p]),
                "paged_attention_decode_shared_prefix": (st, [P(CacheDesc), p, p, p, p, p, i32, p, i32,
                                                              i32, ctypes.c_float, p, p, i32, p, sz,
                                                              p, p]),
                "paged_attention_shared_prefix_workspace_bytes": (sz, [P(CacheDesc), i32, i32, i32, p,
                                                                       p, i32]),
                "pkv_pool_create": (st, [i32, i32, p, P(p)]),
                "pkv_pool_destroy": (None, [p]),
                "pkv_seq_new": (st, [p, P(i32)]),
                "pkv_seq_fork": (st, [p, i32, P(i32)]),
                "pkv_seq_reserve": (st, [p, i32, i32, p, p, P(i32)]),
                "pkv_seq_reserve_tokens": (st, [p, i32, p, i32, p, p, P(i32)]),
                "pkv_seq_new_cached": (st, [p, p, i32, P(i32), P(i32)]),
                "pkv_pool_reserve_batch": (st, [p, p, i32, p, p, p, i32, P(i32), P(i32)]),
                "pkv_seq_cow": (st, [p, i32, i32, p, P(i32)]),
                "pkv_seq_free": (st, [p, i32]),
                "pkv_seq_swap_out": (st, [p, i32, p, i32, P(i32)]),
                "pkv_seq_swap_in": (st, [p, i32, p, i32, P(i32)]),
                "pkv_seq_len": (st, [p, i32, P(i64)]),
                "pkv_seq_block_table": (st, [p, i32, p, i32, P(i32)]),
                "pkv_pool_block_tables": (st, [p, p, i32, p, i32, p, i32]),
                "pkv_pool_refcount": (st, [p, i32, P(i32)]),
                "pkv_pool_free_list": (st, [p, p, i32, P(i32)]),
                "pkv_pool_stats": (st, [p, P(Stats)]),
                "pkv_shared_prefix_groups": (st, [p, i32, i32, p, i32, i32, i32, i32, p, p, P(i32)]),
                "pkv_launch_count": (ctypes.c_uint64, []),
                "pkv_last_error": (ctypes.c_char_p, []),
                "pkv_status_string": (ctypes.c_char_p, [st]),
                "pkv_selftest_wait_timeout": (st, [i32, p, p]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def check(status: int) -> None:
    if status != PKV_OK:
        msg = load().pkv_last_error().decode(errors="replace")
        cls = PoolExhausted if status == 3 else PkvError
        raise cls(status, msg or STATUS_NAMES.get(status, str(status)))
