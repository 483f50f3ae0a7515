"""CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only tests/, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may
import this package.  The library never does, and the oracle never imports the
library: the two share nothing but the seeded input buffers.

``pkv_oracle.c`` holds the arithmetic (plain C, double precision); this module
builds it with gcc on first use and wraps it with numpy arrays.
``bookkeeping.py`` holds the naive model of the block manager.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

from .bookkeeping import BlockPoolModel, PoolExhausted, contiguous_reservation_waste  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pkv_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

F16, BF16 = 0, 1


def build(force: bool = False) -> str:
    """Compile pkv_oracle.c into oracle/_build/liboracle.so (gcc, no fast-math)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                        "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # PKV_ORACLE_LIB selects another build of pkv_oracle.c (the tests use
            # it to check that the pins reject deliberately broken copies).
            lib = ctypes.CDLL(os.environ.get("PKV_ORACLE_LIB") or build())
            p, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            lib.oracle_f16_to_double.restype = dbl
            lib.oracle_f16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_bf16_to_double.restype = dbl
            lib.oracle_bf16_to_double.argtypes = [ctypes.c_uint16]
            lib.oracle_widen.restype = None
            lib.oracle_widen.argtypes = [ctypes.c_int, p, p, i64]
            lib.oracle_attend_dense.restype = None
            lib.oracle_attend_dense.argtypes = [p, p, p, i64, i32, dbl, p, p]
            lib.oracle_paged_decode.restype = ctypes.c_int
            lib.oracle_paged_decode.argtypes = [ctypes.c_int, p, p, p, p, i32, p, i32, i32, i32,
                                                i32, i32, i32, dbl, p, i32, p]
            lib.oracle_paged_decode_split.restype = ctypes.c_int
            lib.oracle_paged_decode_split.argtypes = [ctypes.c_int, p, p, p, p, i32, p, i32, i32,
                                                      i32, i32, i32, i32, dbl, i32, p]
            lib.oracle_paged_prefill.restype = ctypes.c_int
            lib.oracle_paged_prefill.argtypes = [ctypes.c_int, p, p, p, p, i32, p, p, i32, i32,
                                                 i32, i32, i32, i32, dbl, p]
            lib.oracle_append.restype = ctypes.c_int
            lib.oracle_append.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32]
            lib.oracle_copy_blocks.restype = ctypes.c_int
            lib.oracle_copy_blocks.argtypes = [p, p, p, i32, i32, i32, i32, i32]
            lib.oracle_swap_blocks.restype = ctypes.c_int
            lib.oracle_swap_blocks.argtypes = [p, p, p, p, p, i32, i32, i32, i32, i32, i32]
            _lib = lib
    return _lib


def _words(x) -> np.ndarray:
    """16-bit storage words of an fp16 / bf16 tensor or a uint16 array (C-contiguous)."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype in (torch.float16, torch.bfloat16), x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def dtype_code(x) -> int:
    import torch
    return BF16 if x.dtype == torch.bfloat16 else F16


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def widen(words: np.ndarray, dtype: int) -> np.ndarray:
    w = np.ascontiguousarray(words, dtype=np.uint16)
    out = np.empty(w.shape, dtype=np.float64)
    _load().oracle_widen(dtype, _ptr(w), _ptr(out), w.size)
    return out


def attend_dense(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """One query [D] over contiguous K, V [L, D] (float64)."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    L, D = K.shape
    scratch = np.empty(max(L, 1), dtype=np.float64)
    out = np.empty(D, dtype=np.float64)
    _load().oracle_attend_dense(_ptr(q), _ptr(K), _ptr(V), L, D, float(scale), _ptr(scratch),
                                _ptr(out))
    return out


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, seqs=None) -> np.ndarray:
    """Decode attention through the block tables; returns float64 [B, H, D].

    q: fp16/bf16 [B, H, D]; caches: [NB, Hkv, bs, D]; block_tables int32 [B, MB];
    context_lens int32 [B]; seqs: optional subset of sequence indices (others are 0).
    """
    dt = dtype_code(q)
    B, H, D = q.shape
    NB, Hkv, bs, D2 = k_cache.shape
    assert D == D2 and tuple(v_cache.shape) == tuple(k_cache.shape)
    qw, kw, vw = _words(q), _words(k_cache), _words(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.zeros((B, H, D), dtype=np.float64)
    sel = None if seqs is None else np.ascontiguousarray(seqs, dtype=np.int32)
    rc = _load().oracle_paged_decode(dt, _ptr(qw), _ptr(kw), _ptr(vw), _ptr(tables),
                                     tables.shape[1], _ptr(lens), B, H, Hkv, D, bs, NB,
                                     float(scale), None if sel is None else _ptr(sel),
                                     0 if sel is None else len(sel), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode failed ({rc})")
    return out


def paged_decode_split(q, k_cache, v_cache, block_tables, context_lens, scale,
                       partition_size: int) -> np.ndarray:
    dt = dtype_code(q)
    B, H, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    qw, kw, vw = _words(q), _words(k_cache), _words(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    out = np.zeros((B, H, D), dtype=np.float64)
    rc = _load().oracle_paged_decode_split(dt, _ptr(qw), _ptr(kw), _ptr(vw), _ptr(tables),
                                           tables.shape[1], _ptr(lens), B, H, Hkv, D, bs, NB,
                                           float(scale), int(partition_size), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_decode_split failed ({rc})")
    return out


def paged_prefill(q, k_cache, v_cache, block_tables, context_lens, query_start, scale) -> np.ndarray:
    """Causal prefill attention through the block tables; returns float64 [T, H, D].

    q: fp16/bf16 [T, H, D], sequence b's query tokens in rows
    query_start[b] .. query_start[b+1]-1, the last ones of its context_lens[b]
    tokens; caches [NB, Hkv, bs, D]; block_tables int32 [B, MB].
    """
    dt = dtype_code(q)
    T, H, D = q.shape
    NB, Hkv, bs, _ = k_cache.shape
    qw, kw, vw = _words(q), _words(k_cache), _words(v_cache)
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    qs = np.ascontiguousarray(query_start, dtype=np.int32)
    B = len(lens)
    assert len(qs) == B + 1 and qs[-1] == T
    out = np.zeros((T, H, D), dtype=np.float64)
    rc = _load().oracle_paged_prefill(dt, _ptr(qw), _ptr(kw), _ptr(vw), _ptr(tables),
                                      tables.shape[1], _ptr(lens), _ptr(qs), B, H, Hkv, D, bs,
                                      NB, float(scale), _ptr(out))
    if rc != 0:
        raise ValueError(f"oracle_paged_prefill failed ({rc})")
    return out


def append(k_words: np.ndarray, v_words: np.ndarray, key, value, slot_mapping) -> None:
    """In place on uint16 pool arrays [NB, Hkv, bs, D]."""
    NB, Hkv, bs, D = k_words.shape
    kw, vw = _words(key), _words(value)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert k_words.flags.c_contiguous and v_words.flags.c_contiguous
    rc = _load().oracle_append(_ptr(k_words), _ptr(v_words), _ptr(kw), _ptr(vw), _ptr(slots),
                               len(slots), Hkv, D, bs, NB)
    if rc != 0:
        raise ValueError(f"oracle_append failed ({rc})")


def copy_blocks(k_words: np.ndarray, v_words: np.ndarray, block_mapping) -> None:
    NB, Hkv, bs, D = k_words.shape
    pairs = np.ascontiguousarray(block_mapping, dtype=np.int32).reshape(-1, 2)
    rc = _load().oracle_copy_blocks(_ptr(k_words), _ptr(v_words), _ptr(pairs), len(pairs), Hkv,
                                    D, bs, NB)
    if rc != 0:
        raise ValueError(f"oracle_copy_blocks failed ({rc})")


def swap_blocks(k_words: np.ndarray, v_words: np.ndarray, host_k: np.ndarray, host_v: np.ndarray,
                block_list, to_host: bool) -> None:
    """Swap out (to_host) or in whole blocks between uint16 pools [NB, Hkv, bs, D]
    and uint16 host buffers [n, Hkv, bs, D]; all arrays modified in place."""
    NB, Hkv, bs, D = k_words.shape
    blocks = np.ascontiguousarray(block_list, dtype=np.int32)
    for a in (k_words, v_words, host_k, host_v):
        assert a.dtype == np.uint16 and a.flags.c_contiguous
    assert host_k.shape[0] >= len(blocks) and host_v.shape[0] >= len(blocks)
    rc = _load().oracle_swap_blocks(_ptr(k_words), _ptr(v_words), _ptr(host_k), _ptr(host_v),
                                    _ptr(blocks), len(blocks), 1 if to_host else 0, Hkv, D, bs, NB)
    if rc != 0:
        raise ValueError(f"oracle_swap_blocks failed ({rc})")


words = _words
