"""The library's C++ block manager against the oracle's model, bit for bit (no GPU):
the hand-traced golden traces, and long seeded random operation sequences with
tables, slots, copy pairs, reference counts, free lists and statistics compared
after every step."""

import numpy as np
import pytest

from oracle.bookkeeping import BlockPoolModel, PoolExhausted as ModelExhausted
from paged_kv_cache_360_b200 import Pool, PoolExhausted
from tests.trace_player import play


def _lib_pool(nb, bs, order):
    return Pool(nb, bs, order)


@pytest.mark.parametrize("trace", ["bookkeeping_trace.txt", "pool_exhaustion.txt", "swap_trace.txt",
                                   "prefix_cache_trace.txt"])
def test_golden_traces_on_the_library(trace):
    assert play(trace, _lib_pool, PoolExhausted) > 10


def _same(model, pool, live):
    assert pool.free_list() == model.free_list()
    assert pool.stats() == model.stats()
    for sid in live:
        assert pool.table(sid) == model.table(sid)  # empty while swapped out
        assert pool.length(sid) == model.length(sid)
    for b in range(model.num_blocks):
        assert pool.refcount(b) == model.refcount[b]


def _reserve_both(model, pool, sid, n, tokens=None):
    try:
        ms, mp = model.reserve(sid, n) if tokens is None else model.reserve_tokens(sid, tokens)
    except ModelExhausted:
        with pytest.raises(PoolExhausted):
            pool.reserve(sid, n) if tokens is None else pool.reserve_tokens(sid, tokens)
    else:
        ls, lp = pool.reserve(sid, n) if tokens is None else pool.reserve_tokens(sid, tokens)
        assert list(ls) == ms and lp == [tuple(p) for p in mp]


@pytest.mark.parametrize("seed", range(6))
def test_prefix_cached_operation_sequences_match_the_model(seed):
    """Requests built from a few shared prompt stems (so that cache hits, partial
    hits and misses all happen), grown by token ids or by anonymous tokens,
    forked, copied on write, swapped and freed in a seeded random order."""
    rng = np.random.default_rng(900 + seed)
    nb, bs = int(rng.integers(12, 64)), int(rng.choice([1, 2, 4, 8]))
    order = rng.permutation(nb)
    model, pool = BlockPoolModel(nb, bs, order), Pool(nb, bs, order)
    stems = [list(rng.integers(0, 5, size=int(rng.integers(0, 4 * bs + 3)))) for _ in range(3)]
    live = []
    for step in range(400):
        r = rng.random()
        if r < 0.2 or not live:
            prompt = list(stems[int(rng.integers(0, 3))]) + \
                list(rng.integers(0, 5, size=int(rng.integers(0, 2 * bs + 1))))
            a, b = model.new_cached(prompt), pool.new_cached(prompt)
            assert a == b
            live.append(a[0])
            _reserve_both(model, pool, a[0], 0, prompt[a[1]:])
        elif r < 0.3:
            parent = int(rng.choice(live))
            if model.seqs[parent]["swapped"]:
                continue
            a, b = model.fork(parent), pool.fork(parent)
            assert a == b
            live.append(a)
        elif r < 0.65:
            sid = int(rng.choice(live))
            if model.seqs[sid]["swapped"]:
                continue
            n = int(rng.integers(0, 2 * bs + 2))
            anonymous = rng.random() < 0.15
            _reserve_both(model, pool, sid, n,
                          None if anonymous else list(rng.integers(0, 5, size=n)))
        elif r < 0.75:
            sid = int(rng.choice(live))
            if model.seqs[sid]["swapped"]:
                try:
                    mb = model.swap_in(sid)
                except ModelExhausted:
                    with pytest.raises(PoolExhausted):
                        pool.swap_in(sid)
                else:
                    assert pool.swap_in(sid) == mb
            else:
                assert pool.swap_out(sid) == model.swap_out(sid)
        elif r < 0.8:
            sid = int(rng.choice(live))
            nblk = len(model.table(sid))
            if model.seqs[sid]["swapped"] or not nblk:
                continue
            i = int(rng.integers(0, nblk))
            try:
                mp = model.cow(sid, i)
            except ModelExhausted:
                with pytest.raises(PoolExhausted):
                    pool.cow(sid, i)
            else:
                assert pool.cow(sid, i) == mp
        else:
            sid = int(rng.choice(live))
            live.remove(sid)
            model.free_seq(sid)
            pool.free_seq(sid)
        _same(model, pool, live)
    assert model.stats()["cached_blocks"] >= 0


@pytest.mark.parametrize("seed", range(6))
def test_random_operation_sequences_match_the_model(seed):
    rng = np.random.default_rng(100 + seed)
    nb, bs = int(rng.integers(8, 64)), int(rng.choice([1, 2, 4, 16]))
    order = rng.permutation(nb)
    model, pool = BlockPoolModel(nb, bs, order), Pool(nb, bs, order)
    live = []
    for step in range(500):
        r = rng.random()
        if r < 0.12 or not live:
            a, b = model.new_seq(), pool.new_seq()
            assert a == b
            live.append(a)
        elif r < 0.22:
            parent = int(rng.choice(live))
            if model.seqs[parent]["swapped"]:
                continue
            a, b = model.fork(parent), pool.fork(parent)
            assert a == b
            live.append(a)
        elif r < 0.75:
            sid, n = int(rng.choice(live)), int(rng.integers(0, 2 * bs + 2))
            if model.seqs[sid]["swapped"]:
                continue
            try:
                ms, mp = model.reserve(sid, n)
            except ModelExhausted:
                with pytest.raises(PoolExhausted):
                    pool.reserve(sid, n)
            else:
                ls, lp = pool.reserve(sid, n)
                assert list(ls) == ms and lp == [tuple(p) for p in mp]
        elif r < 0.86:
            sid = int(rng.choice(live))
            if model.seqs[sid]["swapped"]:
                try:
                    mb = model.swap_in(sid)
                except ModelExhausted:
                    with pytest.raises(PoolExhausted):
                        pool.swap_in(sid)
                else:
                    assert pool.swap_in(sid) == mb
            else:
                assert pool.swap_out(sid) == model.swap_out(sid)
        elif r < 0.9:
            sid = int(rng.choice(live))
            if model.seqs[sid]["swapped"]:
                continue
            nblk = len(model.table(sid))
            if nblk:
                i = int(rng.integers(0, nblk))
                try:
                    mp = model.cow(sid, i)
                except ModelExhausted:
                    with pytest.raises(PoolExhausted):
                        pool.cow(sid, i)
                else:
                    assert pool.cow(sid, i) == mp
        else:
            sid = int(rng.choice(live))
            live.remove(sid)
            model.free_seq(sid)
            pool.free_seq(sid)
        _same(model, pool, live)


def test_decode_step_export_matches_tables():
    pool = Pool(32, 4, np.random.default_rng(0).permutation(32))
    ids = [pool.new_seq() for _ in range(3)]
    for sid, n in zip(ids, (5, 0, 9)):
        pool.reserve(sid, n)
    tables, lens = pool.block_tables(ids, 4, pad=-1)
    for row, sid in zip(tables, ids):
        t = pool.table(sid)
        assert list(row[:len(t)]) == t and all(x == -1 for x in row[len(t):])
    assert list(lens) == [5, 0, 9]


def test_library_rejects_misuse():
    from paged_kv_cache_360_b200 import PkvError
    with pytest.raises(PkvError):
        Pool(4, 2, [0, 0, 1, 2])                 # not a permutation
    pool = Pool(4, 2)
    with pytest.raises(PkvError):
        pool.reserve(0, 1)                       # unknown sequence
    sid = pool.new_seq()
    pool.free_seq(sid)
    with pytest.raises(PkvError):
        pool.free_seq(sid)                       # already freed
    with pytest.raises(PkvError):
        pool.refcount(9)


def _same_pools(a, b, live):
    assert a.free_list() == b.free_list()
    assert a.stats() == b.stats()
    for sid in live:
        assert a.table(sid) == b.table(sid)
        assert a.length(sid) == b.length(sid)


@pytest.mark.parametrize("seed", range(8))
def test_batched_reserve_equals_the_sequential_calls(seed):
    """pkv_pool_reserve_batch against one pkv_seq_reserve per sequence on a twin
    pool: same slots, copy pairs, tables, free list and statistics, including
    batches that repeat a sequence, write into shared partly filled blocks, and
    run the pool dry half way (the served prefix stands)."""
    rng = np.random.default_rng(1300 + seed)
    nb, bs = int(rng.integers(16, 96)), int(rng.choice([1, 2, 4, 16]))
    order = rng.permutation(nb)
    a, b = Pool(nb, bs, order), Pool(nb, bs, order)
    live, exhausted = [], 0
    for _ in range(250):
        r = rng.random()
        if r < 0.15 or not live:
            sa, sb = a.new_seq(), b.new_seq()
            assert sa == sb
            live.append(sa)
        elif r < 0.27:
            parent = int(live[int(rng.integers(len(live)))])
            ca, cb = a.fork(parent), b.fork(parent)
            assert ca == cb
            live.append(ca)
        elif r < 0.35 and len(live) > 1:
            sid = live.pop(int(rng.integers(len(live))))
            a.free_seq(sid)
            b.free_seq(sid)
        else:
            k = int(rng.integers(1, len(live) + 1))
            seqs = [int(x) for x in rng.choice(live, size=k, replace=True)]
            counts = None if rng.random() < 0.5 else [int(x) for x in rng.integers(0, 2 * bs + 2, size=k)]
            exp_slots, exp_pairs, done, failed = [], [], 0, False
            for i, sid in enumerate(seqs):
                try:
                    s_, p_ = b.reserve(sid, 1 if counts is None else counts[i])
                except PoolExhausted:
                    failed = True
                    break
                exp_slots += [int(x) for x in s_]
                exp_pairs += p_
                done += 1
            if failed:
                exhausted += 1
                with pytest.raises(PoolExhausted) as ei:
                    a.reserve_batch(seqs, counts)
                got_s, got_p = ei.value.slots, ei.value.pairs
                assert ei.value.n_done == done
            else:
                got_s, got_p = a.reserve_batch(seqs, counts)
            assert [int(x) for x in got_s] == exp_slots and got_p == exp_pairs
        _same_pools(a, b, live)
    assert exhausted > 0


def test_batched_reserve_stops_at_a_copy_past_cow_cap():
    import ctypes
    from paged_kv_cache_360_b200 import _lib
    pool = Pool(8, 4, np.arange(8))
    s0 = pool.new_seq()
    pool.reserve(s0, 2)                     # block 0 half full
    s1 = pool.fork(s0)                      # now shared
    s2 = pool.new_seq()
    lib = _lib.load()
    ids = np.array([s2, s1], dtype=np.int32)
    slots = np.empty(2, dtype=np.int64)
    n_cow, n_done = ctypes.c_int32(), ctypes.c_int32()
    st = lib.pkv_pool_reserve_batch(pool._h, ids.ctypes.data_as(ctypes.c_void_p), 2, None,
                                    slots.ctypes.data_as(ctypes.c_void_p), None, 0,
                                    ctypes.byref(n_cow), ctypes.byref(n_done))
    assert st == 1 and n_done.value == 1 and n_cow.value == 0
    assert "cow_cap" in lib.pkv_last_error().decode()
    assert pool.length(s2) == 1 and pool.length(s1) == 2   # s1 untouched
    # with room for the copy, s1 copies its shared half-full block and goes on
    got, pairs = pool.reserve_batch([s1])
    assert len(pairs) == 1 and pairs[0][0] == pool.table(s0)[0] and pool.length(s1) == 3


def test_batched_reserve_on_prefix_cached_sequences():
    """Requests admitted through the prefix cache, then grown by the batched call:
    same slots, pairs, cache statistics and tables as single calls on a twin pool."""
    rng = np.random.default_rng(77)
    nb, bs = 64, 4
    order = rng.permutation(nb)
    a, b = Pool(nb, bs, order), Pool(nb, bs, order)
    stem = [int(x) for x in rng.integers(0, 9, size=10)]
    live = []
    for i in range(5):
        prompt = stem + [int(x) for x in rng.integers(0, 9, size=i)]
        (sid, covered), rb = a.new_cached(prompt), b.new_cached(prompt)
        assert (sid, covered) == rb
        sa, pa = a.reserve_tokens(sid, prompt[covered:])
        sb, pb = b.reserve_tokens(sid, prompt[covered:])
        assert list(sa) == list(sb) and pa == pb
        live.append(sid)
    assert a.stats()["cached_blocks"] > 0
    for _ in range(3):
        counts = [int(x) for x in rng.integers(0, 6, size=len(live))]
        got_s, got_p = a.reserve_batch(live, counts)
        exp_s, exp_p = [], []
        for sid, n in zip(live, counts):
            s_, p_ = b.reserve(sid, n)
            exp_s += [int(x) for x in s_]
            exp_p += p_
        assert [int(x) for x in got_s] == exp_s and got_p == exp_p
        _same_pools(a, b, live)
