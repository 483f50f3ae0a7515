"""Paged KV-cache decode attention for NVIDIA B200 (sm_100a).

A thin Python binding over libpkv.so (include/pkv.h): the functions below have
the C ABI's names and only marshal arguments -- tensor pointers, shapes and the
current CUDA stream.  Every step runs in the library's CUDA kernels or its C++
block manager; there is no CPU fallback.  Device calls require CUDA tensors and
raise if the library is not built.

PyTorch provides device memory and streams only.
"""

from __future__ import annotations

import ctypes

import numpy as np

from . import _lib
from ._lib import PkvError, PoolExhausted  # noqa: F401

__all__ = [
    "paged_kv_append", "copy_blocks", "swap_blocks", "paged_attention_decode",
    "paged_attention_workspace_bytes",
    "paged_attention_decode_static_scratch", "paged_attention_prefill",
    "paged_attention_decode_shared_prefix", "paged_attention_shared_prefix_workspace_bytes",
    "shared_prefix_groups", "Pool",
    "PkvError", "PoolExhausted", "launch_count", "selftest_wait_timeout", "cache_desc",
]


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return _lib.PKV_BF16
    if t.dtype == torch.float16:
        return _lib.PKV_F16
    raise PkvError(2, f"unsupported dtype {t.dtype}: fp16 or bf16 only")


def cache_desc(k_cache) -> _lib.CacheDesc:
    """Descriptor of a pool tensor [num_blocks, num_kv_heads, block_size, head_dim]."""
    if k_cache.dim() != 4:
        raise PkvError(1, "cache must be [num_blocks, num_kv_heads, block_size, head_dim]")
    nb, hkv, bs, d = k_cache.shape
    return _lib.CacheDesc(nb, bs, hkv, d, _dtype_code(k_cache))


def _dev(t, name: str, dtype=None):
    """Device pointer of a contiguous CUDA tensor (raises otherwise)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise PkvError(1, f"{name} must be a CUDA tensor (this library has no CPU path)")
    cur = _torch().cuda.current_device()
    if t.device.index != cur:
        raise PkvError(1, f"{name} is on {t.device} but the current device is cuda:{cur}: "
                          "the library's calls work on the current device only")
    if not t.is_contiguous():
        raise PkvError(1, f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise PkvError(1, f"{name} must be {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = _torch().cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def paged_kv_append(k_cache, v_cache, key, value, slot_mapping, err_flag=None, stream=None):
    """Write key/value [N, Hkv, D] into the pools at slot_mapping (int64 [N]; < 0 skips)."""
    torch = _torch()
    desc = cache_desc(k_cache)
    if tuple(key.shape) != (slot_mapping.shape[0], k_cache.shape[1], k_cache.shape[3]) or \
            key.shape != value.shape or key.dtype != k_cache.dtype or value.dtype != k_cache.dtype:
        raise PkvError(1, "key/value must be [N, num_kv_heads, head_dim] of the cache dtype")
    _lib.check(_lib.load().paged_kv_append(
        ctypes.byref(desc), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(key, "key"),
        _dev(value, "value"), _dev(slot_mapping, "slot_mapping", torch.int64),
        int(slot_mapping.shape[0]), _dev(err_flag, "err_flag", torch.int32), _stream(stream)))


def copy_blocks(k_cache, v_cache, block_mapping, err_flag=None, stream=None):
    """Copy whole blocks src -> dst for each row (src, dst) of block_mapping (int32 [M, 2])."""
    torch = _torch()
    desc = cache_desc(k_cache)
    if block_mapping.dim() != 2 or block_mapping.shape[1] != 2:
        raise PkvError(1, "block_mapping must be [M, 2]")
    _lib.check(_lib.load().copy_blocks(
        ctypes.byref(desc), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(block_mapping, "block_mapping", torch.int32), int(block_mapping.shape[0]),
        _dev(err_flag, "err_flag", torch.int32), _stream(stream)))


def swap_blocks(k_cache, v_cache, host_k, host_v, block_list, to_host: bool, err_flag=None,
                stream=None):
    """Copy whole blocks between the pools and page-locked host buffers
    [n, num_kv_heads, block_size, head_dim]: host[i] = pool[block_list[i]] when
    to_host, else pool[block_list[i]] = host[i].  block_list: int32 CUDA tensor [n]."""
    torch = _torch()
    desc = cache_desc(k_cache)
    n = int(block_list.shape[0])
    for name, t in (("host_k", host_k), ("host_v", host_v)):
        if t.is_cuda or not t.is_pinned() or not t.is_contiguous() or t.dtype != k_cache.dtype:
            raise PkvError(1, f"{name} must be contiguous page-locked host memory of the cache dtype")
        if t.dim() != 4 or t.shape[0] < n or tuple(t.shape[1:]) != tuple(k_cache.shape[1:]):
            raise PkvError(1, f"{name} must be [>= n, num_kv_heads, block_size, head_dim]")
    _lib.check(_lib.load().swap_blocks(
        ctypes.byref(desc), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        ctypes.c_void_p(host_k.data_ptr()), ctypes.c_void_p(host_v.data_ptr()),
        _dev(block_list, "block_list", torch.int32), n, 1 if to_host else 0,
        _dev(err_flag, "err_flag", torch.int32), _stream(stream)))


def paged_attention_workspace_bytes(k_cache, num_seqs: int, num_heads: int,
                                    max_blocks_per_seq: int, partition_size: int = 0) -> int:
    desc = cache_desc(k_cache)
    return int(_lib.load().paged_attention_workspace_bytes(
        ctypes.byref(desc), num_seqs, num_heads, max_blocks_per_seq, partition_size))


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale,
                           partition_size: int = 0, workspace=None, err_flag=None, stream=None):
    """out[b, h] = softmax(scale * q[b, h] . K) V over context_lens[b] tokens read through
    block_tables[b] (int32 [B, MB]).  partition_size 0 splits the batch's work evenly
    over the GPU (the default); > 0 uses fixed partitions of that many tokens.
    `workspace` (uint8 CUDA tensor) is allocated with torch when needed and not
    given.  Returns `out`."""
    torch = _torch()
    desc = cache_desc(k_cache)
    B, H, D = q.shape
    if tuple(out.shape) != (B, H, D) or out.dtype != q.dtype or q.dtype != k_cache.dtype:
        raise PkvError(1, "q and out must be [B, H, D] of the cache dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PkvError(1, "block_tables must be [B, MB] and context_lens [B]")
    MB = int(block_tables.shape[1])
    if workspace is None:
        need = paged_attention_workspace_bytes(k_cache, B, H, MB, partition_size)
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _lib.check(_lib.load().paged_attention_decode(
        ctypes.byref(desc), _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables", torch.int32), MB,
        _dev(context_lens, "context_lens", torch.int32), B, H, ctypes.c_float(scale),
        int(partition_size), _dev(workspace, "workspace"), ws_bytes,
        _dev(err_flag, "err_flag", torch.int32), _stream(stream)))
    return out


def paged_attention_decode_static_scratch(out, q, k_cache, v_cache, block_tables, context_lens,
                                          scale, partition_size: int = 0, err_flag=None,
                                          stream=None):
    """paged_attention_decode for callers that cannot allocate device memory: the
    split path uses the library's fixed 16 MiB scratch array instead of a
    workspace (shapes needing more raise PkvError).  Calls that may run at the
    same time on the GPU race on that array.  Returns `out`."""
    torch = _torch()
    desc = cache_desc(k_cache)
    B, H, D = q.shape
    if tuple(out.shape) != (B, H, D) or out.dtype != q.dtype or q.dtype != k_cache.dtype:
        raise PkvError(1, "q and out must be [B, H, D] of the cache dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PkvError(1, "block_tables must be [B, MB] and context_lens [B]")
    _lib.check(_lib.load().paged_attention_decode_static_scratch(
        ctypes.byref(desc), _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables", torch.int32),
        int(block_tables.shape[1]), _dev(context_lens, "context_lens", torch.int32), B, H,
        ctypes.c_float(scale), int(partition_size), _dev(err_flag, "err_flag", torch.int32),
        _stream(stream)))
    return out


def _group_arrays(group_start, group_shared_blocks):
    gs = np.ascontiguousarray(group_start, dtype=np.int32)
    gb = np.ascontiguousarray(group_shared_blocks, dtype=np.int32)
    n = len(gb)
    if gs.ndim != 1 or gb.ndim != 1 or len(gs) != n + 1:
        raise PkvError(1, "group_start must have one entry more than group_shared_blocks")
    return gs, gb, n


def _ptr_np(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a.size else None


def paged_attention_shared_prefix_workspace_bytes(k_cache, num_seqs: int, num_heads: int,
                                                  max_blocks_per_seq: int, group_start,
                                                  group_shared_blocks) -> int:
    desc = cache_desc(k_cache)
    gs, gb, n = _group_arrays(group_start, group_shared_blocks)
    return int(_lib.load().paged_attention_shared_prefix_workspace_bytes(
        ctypes.byref(desc), num_seqs, num_heads, max_blocks_per_seq, _ptr_np(gs), _ptr_np(gb), n))


def paged_attention_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, context_lens,
                                         scale, group_start, group_shared_blocks, workspace=None,
                                         err_flag=None, stream=None):
    """paged_attention_decode for a batch in which each group of consecutive
    sequences group_start[i] .. group_start[i+1]-1 shares the first
    group_shared_blocks[i] blocks of its tables (host int sequences; see
    shared_prefix_groups).  The shared blocks are attended once per 128 query
    rows on the tensor cores.  `workspace` (uint8 CUDA tensor, 256-byte
    aligned) is allocated with torch when not given.  Returns `out`."""
    torch = _torch()
    desc = cache_desc(k_cache)
    B, H, D = q.shape
    if tuple(out.shape) != (B, H, D) or out.dtype != q.dtype or q.dtype != k_cache.dtype:
        raise PkvError(1, "q and out must be [B, H, D] of the cache dtype")
    if block_tables.dim() != 2 or block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise PkvError(1, "block_tables must be [B, MB] and context_lens [B]")
    MB = int(block_tables.shape[1])
    gs, gb, n = _group_arrays(group_start, group_shared_blocks)
    if workspace is None:
        need = paged_attention_shared_prefix_workspace_bytes(k_cache, B, H, MB, gs, gb)
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _lib.check(_lib.load().paged_attention_decode_shared_prefix(
        ctypes.byref(desc), _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables", torch.int32), MB,
        _dev(context_lens, "context_lens", torch.int32), B, H, ctypes.c_float(scale), _ptr_np(gs),
        _ptr_np(gb), n, _dev(workspace, "workspace"), ws_bytes,
        _dev(err_flag, "err_flag", torch.int32), _stream(stream)))
    return out


def shared_prefix_groups(block_tables, context_lens, block_size: int, min_group_seqs: int = 2,
                         min_shared_blocks: int = 1, max_groups: int = 64):
    """(group_start, group_shared_blocks) for paged_attention_decode_shared_prefix
    from host copies (numpy int32) of a batch's block tables [B, MB] and lengths
    [B]: runs of consecutive sequences whose tables start with the same full
    blocks (pkv_shared_prefix_groups)."""
    tables = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    if tables.ndim != 2 or lens.shape != (tables.shape[0],):
        raise PkvError(1, "block_tables must be [B, MB] and context_lens [B]")
    B, MB = tables.shape
    starts = np.zeros(max_groups + 1, dtype=np.int32)
    shared = np.zeros(max(1, max_groups), dtype=np.int32)
    n = ctypes.c_int32()
    _lib.check(_lib.load().pkv_shared_prefix_groups(
        _ptr_np(tables), B, max(1, MB), _ptr_np(lens), block_size, min_group_seqs,
        min_shared_blocks, max_groups, starts.ctypes.data_as(ctypes.c_void_p),
        shared.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)))
    k = n.value
    return starts[:k + 1], shared[:k]


def paged_attention_prefill(out, q, k_cache, v_cache, block_tables, context_lens, query_start,
                            scale, err_flag=None, stream=None):
    """Causal prefill through the block tables: q and out are [T, H, D] with
    sequence b's query tokens in rows query_start[b] .. query_start[b+1]-1, the
    last ones of its context_lens[b] tokens (already appended).  Returns `out`."""
    torch = _torch()
    desc = cache_desc(k_cache)
    T, H, D = q.shape
    if tuple(out.shape) != (T, H, D) or out.dtype != q.dtype or q.dtype != k_cache.dtype:
        raise PkvError(1, "q and out must be [T, H, D] of the cache dtype")
    B = int(context_lens.shape[0])
    if block_tables.dim() != 2 or block_tables.shape[0] != B or query_start.shape[0] != B + 1:
        raise PkvError(1, "block_tables must be [B, MB], context_lens [B], query_start [B + 1]")
    _lib.check(_lib.load().paged_attention_prefill(
        ctypes.byref(desc), _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"), _dev(block_tables, "block_tables", torch.int32),
        int(block_tables.shape[1]), _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32), B, T, H, ctypes.c_float(scale),
        _dev(err_flag, "err_flag", torch.int32), _stream(stream)))
    return out


def launch_count() -> int:
    """Kernels libpkv has launched in this process."""
    return int(_lib.load().pkv_launch_count())


def selftest_wait_timeout(which, err_flag, stream=None):
    """Run one bounded wait on an mbarrier nothing arrives on (which = 0: the
    decode pipeline wait, 1: the decode abortable wait, 2: the prefill wait);
    it must give up by itself and set DEVERR_WAIT_TIMEOUT in err_flag."""
    torch = _torch()
    _lib.check(_lib.load().pkv_selftest_wait_timeout(
        int(which), _dev(err_flag, "err_flag", torch.int32), _stream(stream)))


class Pool:
    """Host block manager (pkv_pool_* / pkv_seq_*): free pool, block tables,
    reference counts, fork and copy on write.  Host memory only."""

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        lib = _lib.load()
        self.num_blocks, self.block_size = int(num_blocks), int(block_size)
        handle = ctypes.c_void_p()
        order = None
        if free_order is not None:
            self._order = np.ascontiguousarray(free_order, dtype=np.int32)
            order = self._order.ctypes.data_as(ctypes.c_void_p)
        _lib.check(lib.pkv_pool_create(num_blocks, block_size, order, ctypes.byref(handle)))
        self._h = handle
        self._lib = lib

    def close(self):
        if getattr(self, "_h", None):
            self._lib.pkv_pool_destroy(self._h)
            self._h = None

    __del__ = close

    def new_seq(self) -> int:
        sid = ctypes.c_int32()
        _lib.check(self._lib.pkv_seq_new(self._h, ctypes.byref(sid)))
        return sid.value

    def fork(self, parent: int) -> int:
        sid = ctypes.c_int32()
        _lib.check(self._lib.pkv_seq_fork(self._h, parent, ctypes.byref(sid)))
        return sid.value

    def reserve(self, seq: int, n_tokens: int):
        """(slots int64 array, [(src, dst)] copy pairs)."""
        slots = np.empty(max(1, n_tokens), dtype=np.int64)
        pair = np.empty(2, dtype=np.int32)
        n = ctypes.c_int32()
        _lib.check(self._lib.pkv_seq_reserve(self._h, seq, n_tokens,
                                             slots.ctypes.data_as(ctypes.c_void_p),
                                             pair.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)))
        return slots[:n_tokens], ([(int(pair[0]), int(pair[1]))] if n.value else [])

    def reserve_batch(self, seqs, n_tokens=None):
        """One decode step's allocation in one call: reserve(seqs[i], n_tokens[i])
        for every i in order (one token each when n_tokens is None).  Returns
        (slots int64 array of all sequences back to back, [(src, dst)] copy
        pairs).  If sequence i cannot be served, raises PoolExhausted or
        PkvError with .n_done = i and .slots / .pairs of the sequences before
        it, whose reservations stand."""
        ids = np.ascontiguousarray(seqs, dtype=np.int32)
        counts = None if n_tokens is None else np.ascontiguousarray(n_tokens, dtype=np.int32)
        total = len(ids) if counts is None else int(counts.sum())
        slots = np.empty(max(1, total), dtype=np.int64)
        pairs = np.empty((max(1, len(ids)), 2), dtype=np.int32)
        n_cow, n_done = ctypes.c_int32(), ctypes.c_int32()
        st = self._lib.pkv_pool_reserve_batch(
            self._h, ids.ctypes.data_as(ctypes.c_void_p), len(ids),
            None if counts is None else counts.ctypes.data_as(ctypes.c_void_p),
            slots.ctypes.data_as(ctypes.c_void_p), pairs.ctypes.data_as(ctypes.c_void_p), len(ids),
            ctypes.byref(n_cow), ctypes.byref(n_done))
        served = n_done.value if counts is None else int(counts[:n_done.value].sum())
        got_slots = slots[:served]
        got_pairs = [(int(a), int(b)) for a, b in pairs[:n_cow.value]]
        if st != _lib.PKV_OK:
            try:
                _lib.check(st)
            except _lib.PkvError as e:
                e.n_done, e.slots, e.pairs = n_done.value, got_slots, got_pairs
                raise
        return got_slots, got_pairs

    def reserve_tokens(self, seq: int, tokens):
        """reserve() for these token ids, registering the blocks it fills in the
        prefix cache; returns (slots, [(src, dst)] copy pairs)."""
        toks = np.ascontiguousarray(tokens, dtype=np.int32)
        n_tokens = len(toks)
        slots = np.empty(max(1, n_tokens), dtype=np.int64)
        pair = np.empty(2, dtype=np.int32)
        n = ctypes.c_int32()
        _lib.check(self._lib.pkv_seq_reserve_tokens(
            self._h, seq, toks.ctypes.data_as(ctypes.c_void_p), n_tokens,
            slots.ctypes.data_as(ctypes.c_void_p), pair.ctypes.data_as(ctypes.c_void_p),
            ctypes.byref(n)))
        return slots[:n_tokens], ([(int(pair[0]), int(pair[1]))] if n.value else [])

    def new_cached(self, prompt):
        """A new sequence on the longest cached prefix of `prompt`;
        returns (sequence id, tokens covered)."""
        toks = np.ascontiguousarray(prompt, dtype=np.int32)
        sid, covered = ctypes.c_int32(), ctypes.c_int32()
        _lib.check(self._lib.pkv_seq_new_cached(self._h, toks.ctypes.data_as(ctypes.c_void_p),
                                                len(toks), ctypes.byref(sid), ctypes.byref(covered)))
        return sid.value, covered.value

    def cow(self, seq: int, logical_block: int):
        pair = np.empty(2, dtype=np.int32)
        n = ctypes.c_int32()
        _lib.check(self._lib.pkv_seq_cow(self._h, seq, logical_block,
                                         pair.ctypes.data_as(ctypes.c_void_p), ctypes.byref(n)))
        return (int(pair[0]), int(pair[1])) if n.value else None

    def free_seq(self, seq: int) -> None:
        _lib.check(self._lib.pkv_seq_free(self._h, seq))

    def swap_out(self, seq: int):
        """Release the sequence's blocks (preemption); returns them, logical order."""
        n = ctypes.c_int32()
        cap = max(1, len(self.table(seq)))
        out = np.empty(cap, dtype=np.int32)
        _lib.check(self._lib.pkv_seq_swap_out(self._h, seq, out.ctypes.data_as(ctypes.c_void_p), cap,
                                              ctypes.byref(n)))
        return [int(x) for x in out[:n.value]]

    def swap_in(self, seq: int):
        """Fresh blocks for a swapped-out sequence (all or nothing); returns them."""
        n = ctypes.c_int32()
        cap = max(1, -(-self.length(seq) // self.block_size))
        out = np.empty(cap, dtype=np.int32)
        _lib.check(self._lib.pkv_seq_swap_in(self._h, seq, out.ctypes.data_as(ctypes.c_void_p), cap,
                                             ctypes.byref(n)))
        return [int(x) for x in out[:n.value]]

    def length(self, seq: int) -> int:
        n = ctypes.c_int64()
        _lib.check(self._lib.pkv_seq_len(self._h, seq, ctypes.byref(n)))
        return n.value

    def table(self, seq: int):
        n = ctypes.c_int32()
        _lib.check(self._lib.pkv_seq_block_table(self._h, seq, None, 0, ctypes.byref(n)))
        row = np.empty(max(1, n.value), dtype=np.int32)
        _lib.check(self._lib.pkv_seq_block_table(self._h, seq, row.ctypes.data_as(ctypes.c_void_p),
                                                 n.value, ctypes.byref(n)))
        return [int(x) for x in row[:n.value]]

    def block_tables(self, seqs, max_blocks_per_seq: int, pad: int = -1):
        """(int32 [len(seqs), max_blocks_per_seq] tables, int32 [len(seqs)] lengths)."""
        ids = np.ascontiguousarray(seqs, dtype=np.int32)
        tables = np.empty((len(ids), max_blocks_per_seq), dtype=np.int32)
        lens = np.empty(len(ids), dtype=np.int32)
        _lib.check(self._lib.pkv_pool_block_tables(
            self._h, ids.ctypes.data_as(ctypes.c_void_p), len(ids),
            tables.ctypes.data_as(ctypes.c_void_p), max_blocks_per_seq,
            lens.ctypes.data_as(ctypes.c_void_p), pad))
        return tables, lens

    def refcount(self, block: int) -> int:
        r = ctypes.c_int32()
        _lib.check(self._lib.pkv_pool_refcount(self._h, block, ctypes.byref(r)))
        return r.value

    def free_list(self):
        n = ctypes.c_int32()
        _lib.check(self._lib.pkv_pool_free_list(self._h, None, 0, ctypes.byref(n)))
        out = np.empty(max(1, n.value), dtype=np.int32)
        _lib.check(self._lib.pkv_pool_free_list(self._h, out.ctypes.data_as(ctypes.c_void_p),
                                                n.value, ctypes.byref(n)))
        return [int(x) for x in out[:n.value]]

    def stats(self) -> dict:
        s = _lib.Stats()
        _lib.check(self._lib.pkv_pool_stats(self._h, ctypes.byref(s)))
        return {name: int(getattr(s, name)) for name, _ in _lib.Stats._fields_}
