"""GPU parity of the CUDA path against the CPU oracle, through the C ABI.

Append and copy: bit-exact over the whole pool (which also checks that nothing
outside the written slots / blocks changed).  Decode: every output element within
|gpu - oracle| <= 2e-3 + 1e-2 |oracle| of the float64 oracle, on small cases that
span several blocks, partitions and ragged tails, on the edge cases (empty and
one-token contexts, garbage past the last token, bad table entries), and on the
five full-size workloads with the partition size the bench uses.  Block
permutation and copy-on-write must leave the output bit-identical.
"""

import ctypes
import math
import os

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_360_b200 as pkv
from paged_kv_cache_360_b200 import _lib
from paged_kv_cache_360_b200.workloads import (custom_workload, make_workload, random_block_pairs,
                                               random_slot_mapping, normal_tensor)
from tests.gpu_helpers import Dev, compare, ensure_built, oracle_decode, prefix_rows, words

pytestmark = pytest.mark.gpu

DTYPES = [torch.float16, torch.bfloat16]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


def _pool(seed, NB, Hkv, bs, D, dtype):
    rng = np.random.default_rng(seed)
    return (normal_tensor(rng, (NB, Hkv, bs, D), dtype), normal_tensor(rng, (NB, Hkv, bs, D), dtype),
            rng)


# ----------------------------------------------------------------- append / copy

@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("D,bs", [(64, 16), (128, 16), (128, 32), (64, 32)])
def test_append_bit_exact(dtype, D, bs):
    NB, Hkv, N = 37, 8, 150
    k, v, rng = _pool(1, NB, Hkv, bs, D, dtype)
    key, value = normal_tensor(rng, (N, Hkv, D), dtype), normal_tensor(rng, (N, Hkv, D), dtype)
    slots = random_slot_mapping(rng, NB * bs, N, pad_every=7)
    kw, vw = words(k).copy(), words(v).copy()
    oracle.append(kw, vw, key, value, slots)
    kd, vd = k.cuda(), v.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_append(kd, vd, key.cuda(), value.cuda(), torch.from_numpy(slots).cuda(), err_flag=err)
    torch.cuda.synchronize()
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)
    assert err.item() == 0


def test_append_flags_a_slot_past_the_pool():
    NB, Hkv, bs, D = 4, 2, 16, 64
    k, v, rng = _pool(2, NB, Hkv, bs, D, torch.float16)
    key, value = normal_tensor(rng, (3, Hkv, D), torch.float16), normal_tensor(rng, (3, Hkv, D), torch.float16)
    slots = np.array([5, NB * bs + 3, 9], dtype=np.int64)
    kw, vw = words(k).copy(), words(v).copy()
    oracle.append(kw, vw, key[[0, 2]], value[[0, 2]], slots[[0, 2]])
    kd, vd = k.cuda(), v.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_kv_append(kd, vd, key.cuda(), value.cuda(), torch.from_numpy(slots).cuda(), err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & _lib.DEVERR_BAD_SLOT
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("D,bs", [(64, 16), (128, 16), (128, 32)])
def test_copy_blocks_bit_exact(dtype, D, bs):
    NB, Hkv = 64, 8
    k, v, rng = _pool(3, NB, Hkv, bs, D, dtype)
    pairs = random_block_pairs(rng, NB, 31)
    kw, vw = words(k).copy(), words(v).copy()
    oracle.copy_blocks(kw, vw, pairs)
    kd, vd = k.cuda(), v.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks(kd, vd, torch.from_numpy(pairs).cuda(), err_flag=err)
    torch.cuda.synchronize()
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)
    assert err.item() == 0


def test_copy_blocks_flags_an_id_past_the_pool():
    NB, Hkv, bs, D = 8, 2, 16, 64
    k, v, rng = _pool(4, NB, Hkv, bs, D, torch.bfloat16)
    pairs = np.array([[1, 2], [3, NB]], dtype=np.int32)
    kw, vw = words(k).copy(), words(v).copy()
    oracle.copy_blocks(kw, vw, pairs[:1])
    kd, vd = k.cuda(), v.cuda()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.copy_blocks(kd, vd, torch.from_numpy(pairs).cuda(), err_flag=err)
    torch.cuda.synchronize()
    assert err.item() & _lib.DEVERR_BAD_PAIR
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)


# ------------------------------------------------------------------- decode

RAGGED = [1, 2, 15, 16, 17, 31, 32, 33, 100, 257, 511, 512, 513, 1029]


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("D,bs", [(64, 16), (128, 16), (128, 32), (64, 32)])
@pytest.mark.parametrize("group", [1, 4, 8])
def test_decode_ragged_all_partitions(dtype, D, bs, group):
    wl = custom_workload(num_seqs=len(RAGGED), num_heads=2 * group, num_kv_heads=2, head_dim=D,
                         block_size=bs, context_lens=RAGGED, dtype=dtype, seed=group + D + bs)
    dev = Dev(wl)
    ref = oracle_decode(wl)
    for P in (0, bs, 64, 96 if bs == 16 else 128, 512, 1 << 20):
        out = dev.decode(partition_size=P)
        compare(out, ref, what=f"ragged {str(dtype)[6:]} D={D} bs={bs} g={group} P={P}")
        assert dev.err.item() == 0


@pytest.mark.parametrize("dtype", DTYPES)
def test_decode_group_of_sixteen(dtype):
    wl = custom_workload(num_seqs=5, num_heads=32, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=[7, 300, 64, 1000, 129], dtype=dtype, seed=16)
    dev = Dev(wl)
    ref = oracle_decode(wl)
    for P in (0, 128):
        compare(dev.decode(P), ref, what=f"g=16 {str(dtype)[6:]} P={P}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_decode_empty_and_single_token_contexts(dtype):
    wl = custom_workload(num_seqs=4, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=[0, 1, 0, 1], dtype=dtype, seed=5, max_blocks_per_seq=40)
    dev = Dev(wl)
    for P in (0, 64):
        out = dev.decode(P).cpu()
        assert torch.all(out[0] == 0) and torch.all(out[2] == 0)
        for b in (1, 3):
            blk = int(wl.block_tables[b, 0])
            for h in range(8):
                # one token: softmax weight 1, out is that token's value, bit for bit
                assert torch.equal(out[b, h], wl.v_cache[blk, h // 4, 0])


@pytest.mark.parametrize("dtype", DTYPES)
def test_decode_block_permutation_is_bit_identical(dtype):
    wl = custom_workload(num_seqs=6, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[5, 77, 400, 1500, 16, 999], dtype=dtype, seed=9)
    dev = Dev(wl)
    perm = np.random.default_rng(0).permutation(wl.num_blocks)
    k2, v2 = torch.empty_like(dev.k), torch.empty_like(dev.v)
    idx = torch.from_numpy(perm).cuda()
    k2[idx] = dev.k
    v2[idx] = dev.v
    t = wl.block_tables.copy()
    t[t >= 0] = perm[t[t >= 0]]
    t2 = torch.from_numpy(t.astype(np.int32)).cuda()
    for P in (0, 128, 1 << 20):
        assert torch.equal(dev.decode(P), dev.decode(P, tables=t2, k=k2, v=v2))


def test_decode_is_deterministic():
    wl = make_workload(2, seed=3, num_seqs=16)
    dev = Dev(wl)
    a, b = dev.decode(), dev.decode()
    assert torch.equal(a, b)


@pytest.mark.parametrize("dtype", DTYPES)
def test_decode_ignores_garbage_past_the_last_token(dtype):
    lens = [3, 17, 40, 250]
    wl = custom_workload(num_seqs=4, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=lens, dtype=dtype, seed=11)
    for b, L in enumerate(lens):
        blk = int(wl.block_tables[b, (L - 1) // 16])
        wl.k_cache[blk, :, L % 16 or 16:, :] = float("nan")
        wl.v_cache[blk, :, L % 16 or 16:, :] = float("inf")
    dev = Dev(wl)
    ref = oracle_decode(wl)
    for P in (0, 32):
        out = dev.decode(P)
        assert torch.isfinite(out).all()
        compare(out, ref, what=f"garbage tail {str(dtype)[6:]} P={P}")


def test_decode_flags_bad_table_entries_and_lengths():
    wl = custom_workload(num_seqs=3, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=[40, 40, 40], dtype=torch.bfloat16, seed=12)
    dev = Dev(wl)
    bad = wl.block_tables.copy()
    bad[1, 1] = wl.num_blocks + 5
    dev.decode(0, tables=torch.from_numpy(bad).cuda())
    assert dev.err.item() & _lib.DEVERR_BAD_BLOCK_ID
    dev.lens[2] = wl.block_tables.shape[1] * 16 + 1
    dev.decode(0)
    assert dev.err.item() & _lib.DEVERR_BAD_CONTEXT_LEN


def test_decode_rejects_host_tensors_and_small_workspace():
    wl = custom_workload(num_seqs=2, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=[300, 600], dtype=torch.bfloat16, seed=13)
    dev = Dev(wl)
    with pytest.raises(pkv.PkvError):
        pkv.paged_attention_decode(torch.empty_like(wl.q), wl.q, wl.k_cache, wl.v_cache,
                                   torch.from_numpy(wl.block_tables), torch.from_numpy(wl.context_lens),
                                   wl.scale)
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pkv.PkvError) as e:
        pkv.paged_attention_decode(torch.empty_like(dev.q), dev.q, dev.k, dev.v, dev.tables, dev.lens,
                                   wl.scale, partition_size=64, workspace=ws)
    assert e.value.status == 5


# ---------------------------------------------------------- full-size workloads

ORACLE_THREADS = max(1, min(16, os.cpu_count() or 1))


@pytest.mark.parametrize("config", [1, 2, 4, 5])
def test_full_size_workload(config):
    """Every output element of the full-size workload against the oracle, with
    the partition size the bench uses (0 = the balanced schedule; the
    long-context workload's fixed 512-token partitions)."""
    wl = make_workload(config, seed=0)
    dev = Dev(wl)
    P = wl.partition_size
    out = dev.decode(P)
    assert dev.err.item() == 0
    ref = oracle_decode(wl, threads=ORACLE_THREADS)
    mabs, mrel = compare(out, ref, what=f"config {config} ({wl.name}), "
                                         f"{'balanced' if P == 0 else f'fixed P={P}'}")
    assert math.isfinite(mabs)


# -------------------------------------------------------- whole decode step

def _step_both_sides(wl, prefix_blocks_cow):
    """Bookkeeping on each side (library pool / oracle model), then copy, append, decode."""
    bs = wl.block_size
    lib_pool = pkv.Pool(wl.num_blocks, bs, wl.free_order)
    model = oracle.BlockPoolModel(wl.num_blocks, bs, wl.free_order)
    out = {}
    for name, pool in (("lib", lib_pool), ("model", model)):
        s0 = pool.new_seq()
        pool.reserve(s0, wl.prefix_len)
        seqs = [s0] + [pool.fork(s0) for _ in range(wl.num_seqs - 1)]
        pairs = []
        if prefix_blocks_cow is not None:
            for s in seqs:
                p = pool.cow(s, prefix_blocks_cow)
                if p:
                    pairs.append(tuple(p))
        slots = []
        for b, s in enumerate(seqs):
            sl, cp = pool.reserve(s, int(wl.suffix_lens[b]) + 1)
            pairs.extend(tuple(p) for p in cp)
            slots.extend(int(x) for x in sl)
        MB = max(len(pool.table(s)) for s in seqs)
        tables = np.full((len(seqs), MB), -1, dtype=np.int32)
        for i, s in enumerate(seqs):
            t = pool.table(s)
            tables[i, :len(t)] = t
        out[name] = (pairs, slots, tables, np.array([pool.length(s) for s in seqs], dtype=np.int32))
    return out


def _run_step(wl, prefix_blocks_cow):
    sides = _step_both_sides(wl, prefix_blocks_cow)
    pairs, slots, tables, lens = sides["lib"]
    assert [tuple(p) for p in pairs] == [tuple(p) for p in sides["model"][0]]
    assert slots == sides["model"][1]
    assert np.array_equal(tables, sides["model"][2]) and np.array_equal(lens, sides["model"][3])
    # oracle side
    kw, vw = words(wl.k_cache).copy(), words(wl.v_cache).copy()
    mp, ms, mt, ml = sides["model"]
    if mp:
        oracle.copy_blocks(kw, vw, np.array(mp, dtype=np.int32))
    oracle.append(kw, vw, wl.new_key, wl.new_value, np.array(ms, dtype=np.int64))
    # GPU side, through the library
    kd, vd = wl.k_cache.cuda(), wl.v_cache.cuda()
    if pairs:
        pkv.copy_blocks(kd, vd, torch.tensor(pairs, dtype=torch.int32, device="cuda"))
    pkv.paged_kv_append(kd, vd, wl.new_key.cuda(), wl.new_value.cuda(),
                        torch.tensor(slots, dtype=torch.int64, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)
    td, ld = torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda()
    q = wl.q.cuda()
    out = torch.empty_like(q)
    pkv.paged_attention_decode(out, q, kd, vd, td, ld, wl.scale)
    torch.cuda.synchronize()
    k_after = torch.from_numpy(kw.view(np.int16)).view(wl.dtype).reshape(wl.k_cache.shape)
    v_after = torch.from_numpy(vw.view(np.int16)).view(wl.dtype).reshape(wl.v_cache.shape)
    ref = oracle.paged_decode(wl.q, k_after, v_after, mt, ml, wl.scale)
    compare(out, ref, what="decode step")
    return pairs, tables, td, ld, q, kd, vd, out


def test_shared_prefix_step_full_size():
    """Shared-prefix workload: 32 sequences share a 1024-token prefix (64 blocks,
    refcount 32); each takes a private copy of the last prefix block before
    appending (31 copies: the last one finds refcount 1 and keeps the original),
    then its suffix and one new token are appended and the batch is decoded."""
    wl = make_workload(3, seed=0)
    n_prefix = wl.prefix_len // wl.block_size
    pairs, tables, td, ld, q, kd, vd, out = _run_step(wl, n_prefix - 1)
    assert len(pairs) == wl.num_seqs - 1
    # Reading through the original shared block instead of the copies must give
    # the same output bit for bit (a copy leaves content unchanged).
    before = tables.copy()
    before[:, n_prefix - 1] = pairs[0][0]
    out_before = torch.empty_like(q)
    pkv.paged_attention_decode(out_before, q, kd, vd, torch.from_numpy(before).cuda(), ld, wl.scale)
    torch.cuda.synchronize()
    assert torch.equal(out, out_before)


def test_partial_shared_block_copy_on_write():
    """A 20-token prefix (bs 16) leaves a shared, partly filled block: every
    sequence but the last must copy it before its first write."""
    wl = make_workload(3, seed=5, num_seqs=4)
    wl.prefix_len = 20
    wl.suffix_lens = np.array([0, 3, 20, 40], dtype=np.int32)
    n_new = int((wl.suffix_lens + 1).sum())
    rng = np.random.default_rng(1)
    wl.new_key = normal_tensor(rng, (n_new, wl.num_kv_heads, wl.head_dim), wl.dtype)
    wl.new_value = normal_tensor(rng, (n_new, wl.num_kv_heads, wl.head_dim), wl.dtype)
    pairs, *_ = _run_step(wl, None)
    assert len(pairs) == 3


# ------------------------------------------------------------ balanced schedule

@pytest.mark.parametrize("dtype,D,bs,group", [(torch.bfloat16, 128, 16, 4), (torch.float16, 64, 32, 8),
                                              (torch.bfloat16, 128, 32, 8), (torch.bfloat16, 128, 16, 16),
                                              (torch.float16, 64, 16, 1)])
def test_balanced_many_short_and_empty_sequences(dtype, D, bs, group):
    """Hundreds of (sequence, kv head) segments per CTA, some sequences empty."""
    rng = np.random.default_rng(7)
    lens = rng.integers(0, 60, size=700)
    lens[::37] = 0
    wl = custom_workload(num_seqs=700, num_heads=2 * group, num_kv_heads=2, head_dim=D, block_size=bs,
                         context_lens=lens, dtype=dtype, seed=3)
    dev = Dev(wl)
    out = dev.decode(0)
    assert dev.err.item() == 0
    compare(out, oracle_decode(wl), what=f"balanced 700 short {str(dtype)[6:]} D={D} bs={bs} g={group}")
    assert torch.all(out[torch.from_numpy(lens == 0)] == 0)


def test_balanced_one_long_sequence_is_chained_across_ctas():
    wl = custom_workload(num_seqs=1, num_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
                         context_lens=[32768], seed=4)
    dev = Dev(wl)
    out = dev.decode(0)
    assert dev.err.item() == 0
    compare(out, oracle_decode(wl), what="balanced long")


@pytest.mark.parametrize("lens", [[5, 40], [1], [0, 0, 17], [16, 0]])
def test_balanced_fewer_units_than_ctas(lens):
    wl = custom_workload(num_seqs=len(lens), num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=lens, seed=5, max_blocks_per_seq=8)
    dev = Dev(wl)
    out = dev.decode(0)
    assert dev.err.item() == 0
    compare(out, oracle_decode(wl), what=f"balanced {lens}")


def test_balanced_large_batch():
    """More sequences than threads in the prologue's scan (several per thread)."""
    rng = np.random.default_rng(8)
    lens = rng.integers(1, 50, size=3000)
    wl = custom_workload(num_seqs=3000, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=lens, seed=6)
    dev = Dev(wl)
    out = dev.decode(0)
    assert dev.err.item() == 0
    compare(out, oracle_decode(wl), what="balanced large batch")


@pytest.mark.parametrize("config,P", [(4, 0), (5, 512), (2, 512)])
def test_full_size_other_schedule(config, P):
    """The full-size workloads on the schedule the bench does not use by
    default (balanced for the long-context workload, fixed 512-token
    partitions for the others), every output element against the oracle."""
    wl = make_workload(config, seed=0)
    dev = Dev(wl)
    out = dev.decode(P)
    assert dev.err.item() == 0
    compare(out, oracle_decode(wl, threads=ORACLE_THREADS),
            what=f"config {config} ({wl.name}), {'balanced' if P == 0 else f'fixed P={P}'}")


# ------------------------------------------------------------ swap (preemption)

@pytest.mark.parametrize("dtype,D,bs", [(torch.bfloat16, 128, 16), (torch.float16, 64, 32)])
def test_swap_out_and_in_through_the_block_manager(dtype, D, bs):
    """Preempt a sequence (its blocks go to pinned host memory and back to the
    pool), let another sequence reuse the blocks, restore it into fresh blocks:
    the host copy, the pool after restore and the decode output all match the
    oracle, and the output is bit-identical to the output before preemption."""
    rng = np.random.default_rng(11)
    Hkv, H, NB = 4, 16, 64
    k, v, _ = _pool(12, NB, Hkv, bs, D, dtype)
    pool = pkv.Pool(NB, bs, rng.permutation(NB))
    model = oracle.BlockPoolModel(NB, bs, pool.free_list())
    seqs = []
    for L in (300, 77, 150):
        a, b = pool.new_seq(), model.new_seq()
        pool.reserve(a, L)
        model.reserve(b, L)
        seqs.append(a)
    kd, vd = k.cuda(), v.cuda()
    q = normal_tensor(rng, (3, H, D), dtype)
    scale = float(np.float32(1.0 / np.sqrt(D)))

    def decode():
        mb = max(len(pool.table(s)) for s in seqs)
        tables, lens = pool.block_tables(seqs, mb)
        out = torch.empty((3, H, D), dtype=dtype, device="cuda")
        pkv.paged_attention_decode(out, q.cuda(), kd, vd, torch.from_numpy(tables).cuda(),
                                   torch.from_numpy(lens).cuda(), scale)
        torch.cuda.synchronize()
        return out, tables, lens

    before, _, _ = decode()
    victim = seqs[0]
    out_ids = pool.swap_out(victim)
    assert out_ids == model.swap_out(victim)
    host_k = torch.empty((len(out_ids), Hkv, bs, D), dtype=dtype).pin_memory()
    host_v = torch.empty_like(host_k).pin_memory()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.swap_blocks(kd, vd, host_k, host_v, torch.tensor(out_ids, dtype=torch.int32, device="cuda"),
                    to_host=True, err_flag=err)
    torch.cuda.synchronize()
    kw, vw = words(k).copy(), words(v).copy()
    ohk = np.zeros((len(out_ids), Hkv, bs, D), dtype=np.uint16)
    ohv = np.zeros_like(ohk)
    oracle.swap_blocks(kw, vw, ohk, ohv, out_ids, to_host=True)
    assert np.array_equal(words(host_k), ohk) and np.array_equal(words(host_v), ohv)
    # another sequence takes the freed blocks and overwrites them
    other, mo = pool.new_seq(), model.new_seq()
    slots, _ = pool.reserve(other, 200)
    model.reserve(mo, 200)
    junk = normal_tensor(rng, (200, Hkv, D), dtype)
    pkv.paged_kv_append(kd, vd, junk.cuda(), junk.cuda(), torch.from_numpy(slots).cuda())
    oracle.append(kw, vw, junk, junk, slots)
    pool.free_seq(other)
    model.free_seq(mo)
    in_ids = pool.swap_in(victim)
    assert in_ids == model.swap_in(victim)
    pkv.swap_blocks(kd, vd, host_k, host_v, torch.tensor(in_ids, dtype=torch.int32, device="cuda"),
                    to_host=False, err_flag=err)
    oracle.swap_blocks(kw, vw, ohk, ohv, in_ids, to_host=False)
    torch.cuda.synchronize()
    assert err.item() == 0
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)
    after, tables, lens = decode()
    assert torch.equal(before, after)
    k_after = torch.from_numpy(kw.view(np.int16)).view(dtype).reshape(k.shape)
    v_after = torch.from_numpy(vw.view(np.int16)).view(dtype).reshape(v.shape)
    compare(after, oracle.paged_decode(q, k_after, v_after, tables, lens, scale), what="after swap")


def test_swap_blocks_refuses_pageable_host_memory():
    k, v, _ = _pool(13, 4, 2, 16, 64, torch.float16)
    kd, vd = k.cuda(), v.cuda()
    pageable = np.zeros((1, 2, 16, 64), dtype=np.uint16)
    desc = pkv.cache_desc(kd)
    ids = torch.tensor([1], dtype=torch.int32, device="cuda")
    status = _lib.load().swap_blocks(
        ctypes.byref(desc), ctypes.c_void_p(kd.data_ptr()), ctypes.c_void_p(vd.data_ptr()),
        pageable.ctypes.data_as(ctypes.c_void_p), pageable.ctypes.data_as(ctypes.c_void_p),
        ctypes.c_void_p(ids.data_ptr()), 1, 1, None, None)
    assert status == 1
    torch.cuda.synchronize()


# ------------------------------------------------------------ prefix caching

@pytest.mark.parametrize("dtype,D,bs", [(torch.bfloat16, 128, 16), (torch.float16, 64, 32)])
def test_prefix_cached_requests_share_blocks_and_decode_correctly(dtype, D, bs):
    """Three requests with a common system prompt: the second and third start on
    the first one's full prompt blocks (shared, not recomputed), append only
    their own tokens, and decode to the dense oracle over their whole, unpaged
    token rows; the pool matches the oracle's pool after the same appends."""
    rng = np.random.default_rng(21)
    Hkv, H, NB = 2, 8, 48
    system = list(rng.integers(0, 1000, size=3 * bs - 5))
    prompts = [system + list(rng.integers(0, 1000, size=n)) for n in (bs + 3, 2 * bs, 7)]
    pool = pkv.Pool(NB, bs, rng.permutation(NB))
    model = oracle.BlockPoolModel(NB, bs, pool.free_list())
    k0, v0, _ = _pool(22, NB, Hkv, bs, D, dtype)      # stale contents everywhere
    kd, vd = k0.cuda(), v0.cuda()
    kw, vw = words(k0).copy(), words(v0).copy()
    seqs, covered = [], []
    for prompt in prompts:
        sid, n = pool.new_cached(prompt)
        assert (sid, n) == model.new_cached(prompt)
        slots, pairs = pool.reserve_tokens(sid, prompt[n:])
        assert (list(slots), pairs) == model.reserve_tokens(sid, prompt[n:])
        assert pairs == []
        kr, vr = prefix_rows(prompt, Hkv, D, dtype)
        pkv.paged_kv_append(kd, vd, kr[n:].cuda(), vr[n:].cuda(), torch.from_numpy(slots).cuda())
        oracle.append(kw, vw, kr[n:], vr[n:], slots)
        seqs.append(sid)
        covered.append(n)
    # the system prompt's two full blocks are shared by all three requests
    full = (len(system) // bs) * bs
    assert covered == [0, full, full]
    for b in pool.table(seqs[0])[:full // bs]:
        assert pool.refcount(b) == 3
    assert pool.stats() == model.stats()
    torch.cuda.synchronize()
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)

    q = normal_tensor(rng, (3, H, D), dtype)
    mb = max(len(pool.table(s)) for s in seqs)
    tables, lens = pool.block_tables(seqs, mb)
    out = torch.empty((3, H, D), dtype=dtype, device="cuda")
    scale = float(np.float32(1.0 / np.sqrt(D)))
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_attention_decode(out, q.cuda(), kd, vd, torch.from_numpy(tables).cuda(),
                               torch.from_numpy(lens).cuda(), scale, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    code = oracle.BF16 if dtype == torch.bfloat16 else oracle.F16
    ref = np.empty((3, H, D))
    for i, prompt in enumerate(prompts):
        kr, vr = prefix_rows(prompt, Hkv, D, dtype)
        K, V, Q = oracle.widen(words(kr), code), oracle.widen(words(vr), code), \
            oracle.widen(words(q[i]), code)
        for h in range(H):
            hk = h // (H // Hkv)
            ref[i, h] = oracle.attend_dense(Q[h], K[:, hk], V[:, hk], scale)
    compare(out, ref, what="prefix-cached requests")
