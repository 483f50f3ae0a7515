"""paged_attention_decode_static_scratch: the decode for callers that cannot
allocate device memory (a plugin inside an engine whose allocator owns nearly
all of the GPU's memory, or a loop that must never call cudaMalloc).  It keeps
split partials in a fixed 16 MiB array compiled into the library.

Checked through the C ABI against the allocating entry point,
paged_attention_decode, within the tolerance the other decode tests use, on
two calls in a row with different shapes (the array keeps the previous call's
contents, which must not matter).  This file sorts last so that a run that stops
at its first failure has already run every other test."""

import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_360_b200 import _lib, cache_desc
from paged_kv_cache_360_b200.workloads import custom_workload
from tests.gpu_helpers import ATOL, RTOL, Dev, ensure_built

pytestmark = pytest.mark.gpu


def _call_static(dev, partition_size):
    """One call of the no-allocation entry point, straight through ctypes."""
    wl = dev.wl
    desc = cache_desc(dev.k)
    out = torch.full_like(dev.q, float("nan"))
    dev.err.zero_()
    status = _lib.load().paged_attention_decode_static_scratch(
        ctypes.byref(desc), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(dev.q.data_ptr()),
        ctypes.c_void_p(dev.k.data_ptr()), ctypes.c_void_p(dev.v.data_ptr()),
        ctypes.c_void_p(dev.tables.data_ptr()), int(dev.tables.shape[1]),
        ctypes.c_void_p(dev.lens.data_ptr()), wl.num_seqs, wl.num_heads, ctypes.c_float(wl.scale),
        partition_size, ctypes.c_void_p(dev.err.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    torch.cuda.synchronize()
    return status, out


def _close(a, b):
    x = a.float().cpu().double().numpy()
    y = b.float().cpu().double().numpy()
    assert np.all(np.abs(x - y) <= ATOL + RTOL * np.abs(y)), float(np.abs(x - y).max())


def test_static_scratch_matches_the_allocating_entry_point_twice():
    ensure_built()
    cases = [
        (custom_workload(num_seqs=6, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[5, 700, 1500, 16, 999, 3000], seed=41), 256),
        (custom_workload(num_seqs=9, num_heads=16, num_kv_heads=2, head_dim=64, block_size=32,
                         context_lens=[1, 33, 64, 65, 400, 128, 0, 2048, 77],
                         dtype=torch.float16, seed=42), 64),
    ]
    for wl, P in cases:
        dev = Dev(wl)
        expected = dev.decode(partition_size=P)          # allocating entry point
        status, got = _call_static(dev, P)
        assert status == 0, _lib.load().pkv_last_error()
        assert dev.err.item() == 0
        _close(got, expected)


def test_static_scratch_rejects_shapes_beyond_its_size():
    ensure_built()
    wl = custom_workload(num_seqs=2, num_heads=64, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[17, 40], seed=43, max_blocks_per_seq=4096)
    dev = Dev(wl)
    need = _lib.load().paged_attention_workspace_bytes(
        ctypes.byref(cache_desc(dev.k)), wl.num_seqs, wl.num_heads, 4096, 16)
    assert need > _lib.STATIC_SCRATCH_BYTES
    status, _ = _call_static(dev, 16)
    assert status == 5
    assert b"16 MiB" in _lib.load().pkv_last_error()
