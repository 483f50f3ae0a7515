"""Host side of the shared-prefix decode (no GPU): the group helper of the C
ABI against the oracle's model of the same rule, bit for bit, on hand-worked
and random batches; the workspace size; and the host checks of the group
arrays, which reject bad arguments before any CUDA call."""

import ctypes

import numpy as np
import pytest

import paged_kv_cache_360_b200 as pkv
from oracle.bookkeeping import BlockPoolModel, shared_prefix_groups as model_groups
from paged_kv_cache_360_b200 import _build, _lib


@pytest.fixture(scope="module", autouse=True)
def _lib_built():
    _build.build()


def _lib_groups(tables, lens, bs, **kw):
    gs, gb = pkv.shared_prefix_groups(tables, lens, bs, **kw)
    return [int(x) for x in gs], [int(x) for x in gb]


def test_hand_worked_batch():
    # rows 0-2 share blocks 1, 2 (row 2 holds only two full blocks); rows 3-4
    # share 7, 8; row 5 shares nothing with its neighbours
    t = np.array([[1, 2, 3, 4], [1, 2, 3, 9], [1, 2, 5, 6], [7, 8, 9, 9], [7, 8, 0, 0],
                  [3, 3, 3, 3]], dtype=np.int32)
    lens = np.array([64, 64, 40, 64, 33, 64], dtype=np.int32)
    assert _lib_groups(t, lens, 16) == ([0, 3, 5], [2, 2])
    assert model_groups(t, lens, 16) == ([0, 3, 5], [2, 2])
    # three shared blocks needed: rows 0-1 only
    assert _lib_groups(t, lens, 16, min_shared_blocks=3) == ([0, 2], [3])
    assert model_groups(t, lens, 16, min_shared_blocks=3) == ([0, 2], [3])
    # groups of three or more: rows 0-2 only
    assert _lib_groups(t, lens, 16, min_group_seqs=3) == ([0, 3], [2])
    # a gap between kept groups is a group that shares nothing
    t2 = np.array([[1, 2], [1, 2], [5, 6], [7, 8], [7, 8]], dtype=np.int32)
    l2 = np.full(5, 32, dtype=np.int32)
    assert _lib_groups(t2, l2, 16) == ([0, 2, 3, 5], [2, 0, 2])
    assert model_groups(t2, l2, 16) == ([0, 2, 3, 5], [2, 0, 2])
    # room for two entries only: the second group (which needs a gap entry) is dropped
    assert _lib_groups(t2, l2, 16, max_groups=2) == ([0, 2], [2])
    assert model_groups(t2, l2, 16, max_groups=2) == ([0, 2], [2])
    # nothing shared
    assert _lib_groups(t2[2:4], l2[2:4], 16) == ([0], [])


@pytest.mark.parametrize("seed", range(6))
def test_random_forked_batches_match_the_model(seed):
    """Batches built by forking sequences in a block manager (the way shared
    prefixes arise), then growing each on its own."""
    rng = np.random.default_rng(seed)
    bs = int(rng.choice([16, 32]))
    pool = BlockPoolModel(4096, bs)
    seqs = []
    for _ in range(int(rng.integers(1, 6))):
        root = pool.new_seq()
        pool.reserve(root, int(rng.integers(0, 8 * bs)))
        fam = [root] + [pool.fork(root) for _ in range(int(rng.integers(0, 12)))]
        for s in fam:
            pool.reserve(s, int(rng.integers(0, 3 * bs)))
        seqs.extend(fam)
    width = max(1, max(len(pool.table(s)) for s in seqs))
    tables = np.full((len(seqs), width), -1, dtype=np.int32)
    for i, s in enumerate(seqs):
        tables[i, :len(pool.table(s))] = pool.table(s)
    lens = np.array([pool.length(s) for s in seqs], dtype=np.int32)
    for kw in ({}, {"min_group_seqs": 3}, {"min_shared_blocks": 2}, {"max_groups": 3}):
        got = _lib_groups(tables, lens, bs, **kw)
        assert got == model_groups(tables, lens, bs, **kw), kw
        gs, gb = got
        for i, shared in enumerate(gb):   # what the decode relies on
            rows = tables[gs[i]:gs[i + 1]]
            assert np.all(rows[:, :shared] == rows[0, :shared])
            assert np.all(lens[gs[i]:gs[i + 1]] >= shared * bs)


def _desc():
    return _lib.CacheDesc(64, 16, 2, 128, _lib.PKV_BF16)


def test_workspace_bytes_count_the_prefix_partials():
    d = _desc()
    lib = _lib.load()
    gs = (ctypes.c_int32 * 3)(0, 5, 9)
    gb = (ctypes.c_int32 * 2)(9, 0)
    # 9 shared blocks of 16 tokens = 144 tokens = 2 kv tiles, 1 tile per item
    # (few items): 5 sequences x g = 4 heads fit one 128-row tile, so 2 items
    # (chunks) x 2 kv heads tiles of 128 rows; then 5 sequences x 8 heads
    # own-token rows; every row D + 2 floats
    got = lib.paged_attention_shared_prefix_workspace_bytes(ctypes.byref(d), 9, 8, 12, gs, gb, 2)
    if got == 0:
        pytest.skip("no CUDA device to size the balanced part of the workspace")
    plain = lib.paged_attention_workspace_bytes(ctypes.byref(d), 9, 8, 12, 0)
    assert got == ((plain + 255) // 256) * 256 + (2 * 2 * 128 + 5 * 8) * (128 + 2) * 4


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first


@pytest.mark.parametrize("starts,shared,n,status", [
    ([0, 5], [2], 1, 1),          # past num_seqs (4)
    ([2, 2], [2], 1, 1),          # empty group
    ([0, 3, 2], [1, 1], 2, 1),    # decreasing
    ([0, 4], [9], 1, 1),          # more shared blocks than max_blocks_per_seq (8)
    ([0, 4], [-1], 1, 1),
    ([0] * 66, [1] * 65, 65, 2),  # more than 64 groups
])
def test_bad_group_arrays_are_rejected_before_any_launch(starts, shared, n, status):
    lib = _lib.load()
    d = _desc()
    gs = (ctypes.c_int32 * len(starts))(*starts)
    gb = (ctypes.c_int32 * len(shared))(*shared)
    r = lib.paged_attention_decode_shared_prefix(
        ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, 4, 8, ctypes.c_float(0.1), gs, gb,
        n, None, 0, None, None)
    assert r == status, lib.pkv_last_error()


def test_non_power_of_two_group_is_unsupported_when_blocks_are_shared():
    lib = _lib.load()
    d = _desc()
    gs = (ctypes.c_int32 * 2)(0, 4)
    gb = (ctypes.c_int32 * 1)(2)
    r = lib.paged_attention_decode_shared_prefix(
        ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 8, FAKE, 4, 6, ctypes.c_float(0.1), gs, gb,
        1, None, 0, None, None)
    assert r == 2
