"""The bench's accounting, checked on the CPU (no GPU): the causal FLOP count and
the byte counts against brute-force enumeration, and the prefill step's tables
and slots against the oracle's block-manager model."""

import numpy as np
import pytest

import bench
import paged_kv_cache_360_b200 as pkv
from oracle.bookkeeping import BlockPoolModel
from paged_kv_cache_360_b200.workloads import make_prefill_workload, make_workload


def test_prefill_flops_counts_every_visible_pair():
    rng = np.random.default_rng(1)
    lens = rng.integers(1, 300, size=7)
    nq = np.array([rng.integers(0, L + 1) for L in lens])
    qs = np.concatenate([[0], np.cumsum(nq)])
    pairs = sum(L - n + i + 1 for L, n in zip(lens, nq) for i in range(n))
    assert bench.prefill_flops(lens, qs, 8, 64) == pairs * 4 * 8 * 64


def test_decode_bytes_by_enumeration():
    wl = make_workload(1, seed=0, materialize=False)
    lens = wl.context_lens
    per_token = wl.num_kv_heads * wl.head_dim * 2 * 2
    blocks = sum(-(-int(L) // wl.block_size) for L in lens)
    expect = int(lens.sum()) * per_token + 2 * wl.num_seqs * wl.num_heads * wl.head_dim * 2 + \
        4 * blocks + 4 * wl.num_seqs
    assert bench.decode_bytes(lens, wl) == expect


def test_unique_bytes_count_shared_blocks_once():
    wl = make_workload(3, seed=0, materialize=False)
    _, _, tables, lens, _, _ = bench.build_step(wl, bench.library_pool(pkv))
    logical, unique = bench.decode_bytes(lens, wl), bench.unique_decode_bytes(lens, tables, wl)
    per_token = wl.num_kv_heads * wl.head_dim * 4
    slots = set()
    for b, L in enumerate(lens):
        for t in range(int(L)):
            slots.add(int(tables[b, t // wl.block_size]) * wl.block_size + t % wl.block_size)
    assert logical - unique == (int(lens.sum()) - len(slots)) * per_token
    assert unique < logical
    wl2 = make_workload(2, seed=0, materialize=False)
    _, _, t2, l2, _, _ = bench.build_step(wl2, bench.library_pool(pkv))
    assert bench.unique_decode_bytes(l2, t2, wl2) == bench.decode_bytes(l2, wl2)   # no sharing


@pytest.mark.parametrize("name", ["prefill-tiny", "prefill-llama3-8b-layer"])
def test_prefill_step_matches_the_model(name):
    wl = make_prefill_workload(name, seed=2, materialize=False)
    slots, tables, lens = bench.build_prefill_step(wl, bench.library_pool(pkv))
    model = BlockPoolModel(wl.num_blocks, wl.block_size, wl.free_order)
    nq = np.diff(wl.query_start)
    seqs = [model.new_seq() for _ in range(wl.num_seqs)]
    for s, L, n in zip(seqs, wl.context_lens, nq):
        model.reserve(s, int(L - n))
    expect = []
    for s, n in zip(seqs, nq):
        sl, cp = model.reserve(s, int(n))
        assert not cp
        expect.extend(sl)
    assert list(slots) == expect
    for b, s in enumerate(seqs):
        t = model.table(s)
        assert list(tables[b, :len(t)]) == t and all(x == -1 for x in tables[b, len(t):])
    assert list(lens) == list(wl.context_lens)
    assert int(wl.query_start[-1]) == len(slots)


@pytest.mark.parametrize("config", [1, 2, 3, 5])
def test_both_arms_build_the_same_step(config):
    """The reference arm builds the step with the oracle's block-manager model,
    our arm with the library's: pairs, slots, tables and lengths agree exactly."""
    wl = make_workload(config, seed=1, materialize=False)
    ours = bench.build_step(wl, bench.library_pool(pkv))
    ref = bench.build_step(wl, bench.oracle_pool())
    for a, b in zip(ours[:4], ref[:4]):
        assert a.dtype == b.dtype and np.array_equal(a, b)
    assert np.array_equal(ours[3], wl.context_lens)


def test_both_arms_build_the_same_prefill_step():
    wl = make_prefill_workload("prefill-llama3-8b-layer", seed=1, materialize=False)
    ours = bench.build_prefill_step(wl, bench.library_pool(pkv))
    ref = bench.build_prefill_step(wl, bench.oracle_pool())
    for a, b in zip(ours, ref):
        assert a.dtype == b.dtype and np.array_equal(a, b)
