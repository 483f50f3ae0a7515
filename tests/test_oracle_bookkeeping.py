"""Pins for the oracle's block-manager model (no GPU).

The model is tied to the pages' statements, not to itself:

* hand-traced golden traces (tests/golden/bookkeeping_trace.txt,
  pool_exhaustion.txt) derived on paper from the rules of the "PagedAttention"
  ops page (How it works -- The mechanics; Concept -- What it is) and the
  KV-cache lesson's analogy table;
* closed forms: a fresh block is taken exactly when the last one is full, so a
  sequence of n tokens holds ceil(n / block_size) blocks and wastes at most one
  partly filled block (ops page, Concept; lesson: "the only waste left is the
  tail of each request's final block");
* conservation: free + distinct blocks in use == num_blocks after every
  operation; freeing everything returns every block (ops page, Concept);
* sharing: forked sequences point at the same physical blocks with the
  reference count equal to the number of sharers, and a block is copied only
  when a sequence writes into it while it is shared (ops page, How it works and
  At a glance);
* the toy memory map of the lesson's figure, as an illustration.
"""

import math

import numpy as np
import pytest

import oracle
from oracle.bookkeeping import BlockPoolModel, PoolExhausted, contiguous_reservation_waste
from tests.trace_player import GOLDEN, play


def _model(nb, bs, order):
    return BlockPoolModel(nb, bs, order)


def test_golden_trace():
    assert play("bookkeeping_trace.txt", _model, PoolExhausted) > 15


def test_golden_exhaustion_trace():
    assert play("pool_exhaustion.txt", _model, PoolExhausted) > 10


def test_golden_swap_trace():
    assert play("swap_trace.txt", _model, PoolExhausted) > 20


def test_golden_prefix_cache_trace():
    assert play("prefix_cache_trace.txt", _model, PoolExhausted) > 20


def test_prefix_cache_shares_only_identical_prefixes():
    """Two prompts share exactly the full blocks of their common prefix; a block
    is never found under a different prefix."""
    bs = 4
    pool = BlockPoolModel(64, bs)
    a = pool.new_seq()
    prompt = list(range(100, 123))                 # 23 tokens: 5 full blocks + 3
    pool.reserve_tokens(a, prompt)
    assert pool.stats()["cached_blocks"] == 5
    for n_same in range(0, 23):
        other = prompt[:n_same] + [7] * (23 - n_same)
        sid, covered = pool.new_cached(other)
        assert covered == (n_same // bs) * bs
        assert pool.table(sid) == pool.table(a)[:n_same // bs]
        pool.free_seq(sid)
    # the same block contents after a different first block are not a hit
    b = pool.new_seq()
    pool.reserve_tokens(b, [9, 9, 9, 9] + prompt[4:8])
    sid, covered = pool.new_cached([1, 2, 3, 4] + prompt[4:8])
    assert covered == 0
    # dropping a block drops every entry chained below it
    pool.free_seq(a)
    assert pool.stats()["cached_blocks"] == 2      # b's two blocks
    sid, covered = pool.new_cached(prompt)
    assert covered == 0


def test_prefix_cache_random_operations_keep_invariants():
    rng = np.random.default_rng(9)
    pool = BlockPoolModel(48, 2, rng.permutation(48))
    live = []
    vocab = [1, 2, 3]
    for _ in range(600):
        r = rng.random()
        try:
            if r < 0.2 or not live:
                prompt = [int(x) for x in rng.choice(vocab, size=int(rng.integers(0, 9)))]
                sid, covered = pool.new_cached(prompt)
                assert covered % 2 == 0 and covered <= len(prompt)
                live.append(sid)
                pool.reserve_tokens(sid, prompt[covered:])
            elif r < 0.6:
                sid = int(rng.choice(live))
                if not pool.seqs[sid]["swapped"]:
                    pool.reserve_tokens(sid, [int(x) for x in rng.choice(vocab, size=int(rng.integers(1, 4)))])
            elif r < 0.7:
                sid = int(rng.choice(live))
                if not pool.seqs[sid]["swapped"]:
                    live.append(pool.fork(sid))
            else:
                sid = int(rng.choice(live))
                live.remove(sid)
                pool.free_seq(sid)
        except PoolExhausted:
            pass
        _check_invariants_with_swaps(pool)
        # every entry names a block in use whose tokens match its name
        for (prev, toks), blk in pool.cache.items():
            assert pool.refcount[blk] > 0
            holders = [s for s in pool.seqs.values() if blk in s["blocks"] and s["tokens"] is not None]
            for s in holders:
                i = s["blocks"].index(blk)
                if len(s["tokens"]) >= (i + 1) * 2:
                    assert tuple(s["tokens"][2 * i:2 * i + 2]) == toks
                    assert (s["blocks"][i - 1] if i else -1) == prev


def test_swap_round_trip_keeps_length_and_conserves_the_pool():
    """A preempted sequence gives every block back; restoring it takes exactly
    ceil(len / bs) fresh blocks and it can grow again afterwards."""
    pool = BlockPoolModel(20, 4, np.random.default_rng(1).permutation(20))
    a, b = pool.new_seq(), pool.new_seq()
    pool.reserve(a, 13)
    pool.reserve(b, 5)
    shared = pool.fork(a)                          # a's blocks are shared with `shared`
    free_before = len(pool.free)
    out = pool.swap_out(a)
    assert out == pool.table(shared)               # a held the same blocks
    assert len(pool.free) == free_before           # still held by `shared`
    pool.free_seq(shared)
    assert len(pool.free) == free_before + 4
    _check_invariants_with_swaps(pool)
    back = pool.swap_in(a)
    assert len(back) == 4 and pool.length(a) == 13 and all(pool.refcount[x] == 1 for x in back)
    slots, pairs = pool.reserve(a, 4)
    assert pairs == [] and len(pool.table(a)) == math.ceil(17 / 4)
    _check_invariants_with_swaps(pool)
    with pytest.raises(ValueError):
        pool.swap_in(a)                            # not swapped
    pool.swap_out(b)
    with pytest.raises(ValueError):
        pool.reserve(b, 1)                         # swapped sequences cannot grow


def _check_invariants_with_swaps(pool):
    in_use = set()
    for s in pool.seqs.values():
        if s["swapped"]:
            assert s["blocks"] == []
        else:
            assert len(s["blocks"]) == math.ceil(s["len"] / pool.block_size)
        in_use.update(s["blocks"])
    assert len(pool.free) + len(in_use) == pool.num_blocks


@pytest.mark.parametrize("bs", [1, 4, 16])
def test_fresh_block_exactly_when_last_is_full(bs):
    pool = BlockPoolModel(64, bs)
    sid = pool.new_seq()
    for n in range(1, 200):
        before = len(pool.table(sid))
        slots, pairs = pool.reserve(sid, 1)
        took = len(pool.table(sid)) - before
        assert took == (1 if (n - 1) % bs == 0 else 0)
        assert pairs == []
        assert len(pool.table(sid)) == math.ceil(n / bs)
        if n >= 64 * bs:
            break


def _check_invariants(pool):
    in_use = set()
    for s in pool.seqs.values():
        assert len(s["blocks"]) == math.ceil(s["len"] / pool.block_size)
        in_use.update(s["blocks"])
    assert len(pool.free) + len(in_use) == pool.num_blocks
    assert set(pool.free).isdisjoint(in_use)
    for b in range(pool.num_blocks):
        holders = sum(s["blocks"].count(b) for s in pool.seqs.values())
        assert pool.refcount[b] == holders


@pytest.mark.parametrize("seed", range(4))
def test_random_operations_keep_invariants(seed):
    rng = np.random.default_rng(seed)
    nb, bs = 40, 4
    pool = BlockPoolModel(nb, bs, rng.permutation(nb))
    live = []
    for _ in range(400):
        r = rng.random()
        try:
            if r < 0.15 or not live:
                live.append(pool.new_seq())
            elif r < 0.25:
                live.append(pool.fork(int(rng.choice(live))))
            elif r < 0.8:
                sid = int(rng.choice(live))
                before = pool.stats()
                slots, pairs = pool.reserve(sid, int(rng.integers(0, 7)))
                assert len(pairs) <= 1
                if pairs:
                    src, dst = pairs[0]
                    assert pool.refcount[dst] == 1 and dst in pool.table(sid)
                    assert src not in pool.table(sid)
                assert pool.stats()["live_tokens"] == before["live_tokens"] + len(slots)
            else:
                sid = int(rng.choice(live))
                live.remove(sid)
                pool.free_seq(sid)
        except PoolExhausted:
            pass
        _check_invariants(pool)
        st = pool.stats()
        # waste: at most one partly filled block per sequence
        assert st["allocated_slots"] - st["live_slots"] <= (bs - 1) * max(1, st["num_seqs"])
    for sid in list(live):
        pool.free_seq(sid)
    assert sorted(pool.free) == list(range(nb))


def test_waste_bound_on_unshared_sequences():
    rng = np.random.default_rng(3)
    bs = 16
    lens = rng.integers(1, 300, size=50)
    pool = BlockPoolModel(int(sum(math.ceil(x / bs) for x in lens)), bs)
    for L in lens:
        pool.reserve(pool.new_seq(), int(L))
    st = pool.stats()
    assert st["free_blocks"] == 0
    assert st["allocated_slots"] - st["live_slots"] == sum(math.ceil(x / bs) * bs - x for x in lens)
    assert st["allocated_slots"] - st["live_slots"] <= (bs - 1) * len(lens)


def test_fork_shares_blocks_and_cow_copies_exactly_one():
    pool = BlockPoolModel(32, 4)
    parent = pool.new_seq()
    pool.reserve(parent, 10)                       # blocks: 3, last one half full
    kids = [pool.fork(parent) for _ in range(3)]
    for k in kids:
        assert pool.table(k) == pool.table(parent)
    assert all(pool.refcount[b] == 4 for b in pool.table(parent))
    free_before = len(pool.free)
    slots, pairs = pool.reserve(kids[0], 1)        # write into the shared partial block
    assert len(pairs) == 1 and pairs[0][0] == pool.table(parent)[2]
    assert len(pool.free) == free_before - 1
    assert pool.table(kids[0])[:2] == pool.table(parent)[:2]   # the rest stays shared
    assert pool.refcount[pool.table(parent)[0]] == 4
    assert pool.refcount[pool.table(parent)[2]] == 3
    # writing past a full shared block takes a fresh block, no copy
    full = BlockPoolModel(8, 4)
    a = full.new_seq()
    full.reserve(a, 8)
    b = full.fork(a)
    _, pairs = full.reserve(b, 1)
    assert pairs == []


def test_explicit_cow_of_a_shared_block():
    pool = BlockPoolModel(16, 4)
    a = pool.new_seq()
    pool.reserve(a, 8)
    b = pool.fork(a)
    src = pool.table(a)[1]
    pair = pool.cow(b, 1)
    assert pair == (src, pool.table(b)[1]) and pool.refcount[src] == 1
    assert pool.cow(a, 1) is None                  # now private to a: nothing to copy


def test_toy_memory_map_illustration():
    spec = {}
    for raw in open(f"{GOLDEN}/toy_memory_map.txt"):
        line = raw.split("#", 1)[0].split()
        if line:
            spec.setdefault(line[0], []).append(line[1:])
    slots = int(spec["slots"][0][0])
    bs = int(spec["block_size"][0][0])
    reqs = [(int(r[1]), int(r[3])) for r in spec["request"]]
    reserved = sum(res for _, res in reqs)
    assert slots - reserved == int(spec["contiguous_free"][0][0])
    pool = BlockPoolModel(slots, bs)
    for n, _ in reqs:
        pool.reserve(pool.new_seq(), n)
    assert pool.stats()["free_blocks"] == int(spec["paged_free"][0][0])


def check_contiguous_reservation_waste(fn):
    """Exact pins of the slab scheme's accounting (``fn`` is the function under
    test, so that the mutation tests can hand in broken copies):

    * the lesson's toy memory map (tests/golden/toy_memory_map.txt): twelve
      slots of four tokens; A holds 14 tokens in a reservation of 6 slots, B 9
      tokens in 5 slots, so the contiguous row leaves exactly 1 slot free;
    * a batch worked by hand with one request longer than its reservation (a
      slab holds at most what was reserved): lengths 5, 12, 3, 0 with 8 tokens
      reserved each give 32 reserved, 5 + 8 + 3 + 0 = 16 live, 16 wasted;
    * an empty batch reserves nothing.
    """
    spec = {}
    for raw in open(f"{GOLDEN}/toy_memory_map.txt"):
        line = raw.split("#", 1)[0].split()
        if line:
            spec.setdefault(line[0], []).append(line[1:])
    slots, bs = int(spec["slots"][0][0]), int(spec["block_size"][0][0])
    lengths = [int(r[1]) for r in spec["request"]]
    reserve = [int(r[3]) * bs for r in spec["request"]]
    toy = fn(lengths, reserve)
    assert toy == {"reserved_slots": 44, "live_slots": 23, "wasted_slots": 21}
    assert (slots * bs - toy["reserved_slots"]) // bs == int(spec["contiguous_free"][0][0]) == 1
    assert fn([5, 12, 3, 0], 8) == {"reserved_slots": 32, "live_slots": 16, "wasted_slots": 16}
    assert fn([], 8) == {"reserved_slots": 0, "live_slots": 0, "wasted_slots": 0}


def test_contiguous_reservation_waste_exact():
    check_contiguous_reservation_waste(contiguous_reservation_waste)


def test_fragmentation_context_on_synthetic_lengths():
    """Context only (not a pin): paged waste vs a max-length slab per request on
    the long-context mixes; the glossary page quotes <4 % vs 60-80 %."""
    from paged_kv_cache_360_b200.workloads import make_workload
    for cfg, reserve in ((2, 4096), (5, 8192)):
        wl = make_workload(cfg, materialize=False)
        bs = wl.block_size
        lens = [int(x) for x in wl.context_lens]
        paged = sum(math.ceil(x / bs) * bs - x for x in lens) / sum(math.ceil(x / bs) * bs
                                                                     for x in lens)
        slab = contiguous_reservation_waste(lens, reserve)
        assert paged < 0.04 and slab["wasted_slots"] / slab["reserved_slots"] > 0.4
