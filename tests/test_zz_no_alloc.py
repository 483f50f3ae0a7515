"""paged_attention_decode_static_scratch: the decode for callers that cannot
allocate device memory (a plugin inside an engine whose allocator owns nearly
all of the GPU's memory, or a loop that must never call cudaMalloc).  It keeps
split partials in a fixed 16 MiB array compiled into the library.

Checked through the C ABI against the allocating entry point,
paged_attention_decode: both run the same kernels in the same order, so their
outputs must be identical bit for bit (which is within the tolerance the other
decode tests use), and both are checked against the oracle.  The calls come in
a row with different shapes and schedules -- fixed partitions, then the default
balanced schedule, whose merge reads per-CTA descriptors from the array -- so
each call finds the previous call's contents in the array, which must not
matter.  This file sorts last so that a run that stops at its first failure has
already run every other test."""

import ctypes

import pytest
import torch

from paged_kv_cache_360_b200 import _lib, cache_desc
from paged_kv_cache_360_b200.workloads import custom_workload
from tests.gpu_helpers import Dev, compare, ensure_built, oracle_decode

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


def test_static_scratch_matches_the_allocating_entry_point_in_a_row():
    ensure_built()
    cases = [
        (custom_workload(num_seqs=6, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[5, 700, 1500, 16, 999, 3000], seed=41), 256),
        (custom_workload(num_seqs=9, num_heads=16, num_kv_heads=2, head_dim=64, block_size=32,
                         context_lens=[1, 33, 64, 65, 400, 128, 0, 2048, 77],
                         dtype=torch.float16, seed=42), 64),
        # balanced (the default schedule) after two split calls: sequences
        # straddle CTAs, so the chain merge reads partials and descriptors
        # from the array the previous calls left behind
        (custom_workload(num_seqs=5, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[9000, 1, 4000, 0, 2500], seed=44), 0),
        (custom_workload(num_seqs=6, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[5, 700, 1500, 16, 999, 3000], seed=41), 0),
    ]
    for wl, P in cases:
        dev = Dev(wl)
        expected = dev.decode(partition_size=P)          # allocating entry point
        assert dev.err.item() == 0
        status, got = _call_static(dev, P)
        assert status == 0, _lib.load().pkv_last_error()
        assert dev.err.item() == 0
        assert torch.equal(got, expected), f"P={P}: differs from paged_attention_decode"
        compare(got, oracle_decode(wl), what=f"static scratch, P={P}")


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
