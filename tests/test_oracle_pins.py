"""Pins for the CPU oracle's attention, append and copy (no GPU).

Each check ties the oracle to something other than itself:

* torch's dtype conversion for every fp16 / bf16 bit pattern (widening);
* torch's ``scaled_dot_product_attention`` in float64 with ``enable_gqa`` (the
  textbook softmax attention, query head h reading kv head h // g) over a slab
  obtained by *reshaping* a pool whose blocks are in logical order, so the test
  never re-types the oracle's index arithmetic;
* closed forms (one token, all-zero keys, zero query, a single non-zero key);
* block-permutation invariance, bit for bit ("PagedAttention" ops page, How it
  works: reading through the block table makes non-contiguous storage
  transparent to the math);
* the log-sum-exp split identity for several partition sizes;
* byte round trips for append and copy, with every untouched slot checked.

``test_oracle_mutations.py`` re-runs this file against deliberately broken
builds of the oracle and requires each of them to fail here.
"""

import math

import numpy as np
import pytest
import torch

import oracle

RTOL = 1e-12


def _pool(rng, NB, Hkv, bs, D, dtype):
    x = torch.from_numpy(rng.standard_normal((NB, Hkv, bs, D), dtype=np.float32)).to(dtype)
    y = torch.from_numpy(rng.standard_normal((NB, Hkv, bs, D), dtype=np.float32)).to(dtype)
    return x, y


def _identity_case(seed, B=2, H=4, Hkv=2, D=8, bs=4, lens=(37, 9), dtype=torch.bfloat16):
    """Pool laid out in logical order: sequence b owns blocks [b*MB, (b+1)*MB)."""
    rng = np.random.default_rng(seed)
    MB = max(-(-x // bs) for x in lens)
    NB = B * MB
    k, v = _pool(rng, NB, Hkv, bs, D, dtype)
    q = torch.from_numpy(rng.standard_normal((B, H, D), dtype=np.float32)).to(dtype)
    tables = np.arange(NB, dtype=np.int32).reshape(B, MB)
    return q, k, v, tables, np.asarray(lens, dtype=np.int32), MB


def _slab(cache, b, MB, L):
    """Keys (or values) of sequence b as [Hkv, L, D] -- a reshape, no index arithmetic."""
    seq = cache[b * MB:(b + 1) * MB]              # [MB, Hkv, bs, D]
    Hkv, D = seq.shape[1], seq.shape[3]
    return seq.permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :L, :].to(torch.float64)


def _sdpa(q_bh, K, V, scale):
    """torch SDPA, float64, one query per head, grouped kv heads."""
    out = torch.nn.functional.scaled_dot_product_attention(
        q_bh[None, :, None, :], K[None], V[None], scale=scale, enable_gqa=True)
    return out[0, :, 0, :]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_widening_matches_torch_for_every_bit_pattern(dtype):
    allw = np.arange(65536, dtype=np.uint16)
    code = oracle.BF16 if dtype == torch.bfloat16 else oracle.F16
    ours = oracle.widen(allw, code)
    ref = torch.from_numpy(allw.view(np.int16)).view(dtype).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (8, 2), (8, 1)])
def test_brute_force_matches_sdpa_float64(dtype, H, Hkv):
    q, k, v, tables, lens, MB = _identity_case(seed=H * 10 + Hkv, H=H, Hkv=Hkv, dtype=dtype,
                                               lens=(37, 9))
    scale = 1.0 / math.sqrt(8)
    out = oracle.paged_decode(q, k, v, tables, lens, scale)
    for b, L in enumerate(lens):
        ref = _sdpa(q[b].to(torch.float64), _slab(k, b, MB, L), _slab(v, b, MB, L), scale)
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=RTOL, atol=1e-14)


def test_single_token_returns_its_value_exactly():
    q, k, v, tables, lens, MB = _identity_case(seed=3, lens=(1, 1))
    out = oracle.paged_decode(q, k, v, tables, lens, 0.3)
    for b in range(2):
        for h in range(4):
            assert np.array_equal(out[b, h], _slab(v, b, MB, 1)[h // 2, 0].numpy())


def test_zero_keys_and_zero_query_give_the_mean_of_values():
    q, k, v, tables, lens, MB = _identity_case(seed=4, lens=(23, 40))
    kz = torch.zeros_like(k)
    out_k = oracle.paged_decode(q, kz, v, tables, lens, 0.5)
    out_q = oracle.paged_decode(torch.zeros_like(q), k, v, tables, lens, 0.5)
    for b, L in enumerate(lens):
        mean = _slab(v, b, MB, L).mean(dim=1).numpy()      # [Hkv, D]
        expect = np.repeat(mean, 2, axis=0)                  # query head h -> kv head h // 2
        np.testing.assert_allclose(out_k[b], expect, rtol=RTOL, atol=1e-14)
        np.testing.assert_allclose(out_q[b], expect, rtol=RTOL, atol=1e-14)


def test_single_nonzero_key_closed_form():
    """Only key j is non-zero: s_j = c, every other score 0, so
    out = (e^c V_j + sum_{t != j} V_t) / (e^c + L - 1)."""
    q, k, v, tables, lens, MB = _identity_case(seed=5, lens=(19, 19), Hkv=4, H=4)
    j, L = 7, 19
    k = torch.zeros_like(k)
    kv = torch.tensor([0.5, -1.0, 2.0, 0.25, 1.5, -0.75, 1.0, 3.0], dtype=k.dtype)
    # token j of sequence 0 sits in block j // bs of the logical-order pool
    k[j // 4, :, j % 4, :] = kv
    scale = 0.5
    out = oracle.paged_decode(q, k, v, tables, lens, scale)
    V = _slab(v, 0, MB, L).numpy()
    for h in range(4):
        c = scale * float(torch.dot(q[0, h].double(), kv.double()))
        others = V[h].sum(axis=0) - V[h, j]
        expect = (math.exp(c) * V[h, j] + others) / (math.exp(c) + L - 1)
        np.testing.assert_allclose(out[0, h], expect, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_block_permutation_invariance_is_bit_exact(seed):
    q, k, v, tables, lens, MB = _identity_case(seed=10 + seed, lens=(37, 22))
    base = oracle.paged_decode(q, k, v, tables, lens, 0.35)
    perm = np.random.default_rng(seed).permutation(k.shape[0])
    k2, v2 = torch.empty_like(k), torch.empty_like(v)
    k2[perm] = k
    v2[perm] = v
    t2 = perm[tables].astype(np.int32)
    moved = oracle.paged_decode(q, k2, v2, t2, lens, 0.35)
    assert np.array_equal(base, moved)


def test_contiguous_slab_equality():
    """Paged read of a shuffled pool == dense attention over the logical slab, bit for bit."""
    q, k, v, tables, lens, MB = _identity_case(seed=21, lens=(33, 12))
    perm = np.random.default_rng(7).permutation(k.shape[0])
    k2, v2 = torch.empty_like(k), torch.empty_like(v)
    k2[perm] = k
    v2[perm] = v
    paged = oracle.paged_decode(q, k2, v2, perm[tables].astype(np.int32), lens, 0.4)
    for b, L in enumerate(lens):
        K, V = _slab(k, b, MB, L).numpy(), _slab(v, b, MB, L).numpy()
        for h in range(4):
            dense = oracle.attend_dense(q[b, h].double().numpy(), K[h // 2], V[h // 2], 0.4)
            assert np.array_equal(paged[b, h], dense)


def test_empty_context_gives_zeros():
    q, k, v, tables, lens, MB = _identity_case(seed=8, lens=(0, 5))
    out = oracle.paged_decode(q, k, v, tables, lens, 0.3)
    assert np.all(out[0] == 0.0) and np.any(out[1] != 0.0)


@pytest.mark.parametrize("P", [1, 4, 16, 37, 4096])
def test_split_identity(P):
    q, k, v, tables, lens, MB = _identity_case(seed=30, lens=(61, 17), D=16, bs=8)
    mono = oracle.paged_decode(q, k, v, tables, lens, 0.25)
    split = oracle.paged_decode_split(q, k, v, tables, lens, 0.25, P)
    np.testing.assert_allclose(split, mono, rtol=1e-12, atol=1e-14)


def test_sequence_subset_matches_full():
    q, k, v, tables, lens, MB = _identity_case(seed=31, lens=(13, 29))
    full = oracle.paged_decode(q, k, v, tables, lens, 0.3)
    part = oracle.paged_decode(q, k, v, tables, lens, 0.3, seqs=[1])
    assert np.array_equal(part[1], full[1]) and np.all(part[0] == 0)


def test_sequence_index_outside_the_batch_is_rejected():
    """A listed sequence index outside 0 .. B-1 returns -2 before anything of
    that sequence is read.  The call goes straight to the C function with one
    spare (valid) length and one spare output row behind the batch, so an
    oracle that skipped the check would compute that row and return 0 instead
    of faulting."""
    import ctypes
    q, k, v, tables, lens, MB = _identity_case(seed=32, lens=(13, 29))
    B, H, D = q.shape
    NB, Hkv, bs, _ = k.shape
    lens_spare = np.array(list(lens) + [5], dtype=np.int32)
    tables_spare = np.concatenate([tables, tables[:1]]).astype(np.int32)
    q_spare = np.ascontiguousarray(np.concatenate([oracle.words(q), oracle.words(q)[:1]]))
    kw, vw = oracle.words(k), oracle.words(v)
    out = np.zeros((B + 1, H, D), dtype=np.float64)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    for bad in (B, -1):
        sel = np.array([0, bad], dtype=np.int32)
        out[:] = 0
        rc = oracle._load().oracle_paged_decode(
            oracle.BF16, ptr(q_spare[1:] if bad < 0 else q_spare), ptr(kw), ptr(vw),
            ptr(tables_spare[1:] if bad < 0 else tables_spare), MB,
            ptr(lens_spare[1:] if bad < 0 else lens_spare), B, H, Hkv, D, bs, NB, 0.3, ptr(sel),
            len(sel), ptr(out[1:] if bad < 0 else out))
        assert rc == -2, (bad, rc)
    with pytest.raises(ValueError):
        oracle.paged_decode(q, k, v, tables, lens, 0.3, seqs=[0, B])


def _kv_rows(words, Hkv, D):
    """Pool [NB, Hkv, bs, D] as [Hkv, NB*bs, D]: row s is slot s (a reshape)."""
    NB, _, bs, _ = words.shape
    return words.transpose(1, 0, 2, 3).reshape(Hkv, NB * bs, D)


def test_append_round_trip_and_canaries():
    rng = np.random.default_rng(40)
    NB, Hkv, bs, D, N = 6, 2, 4, 8, 9
    k, v = _pool(rng, NB, Hkv, bs, D, torch.float16)
    kw, vw = oracle.words(k).copy(), oracle.words(v).copy()
    k0, v0 = kw.copy(), vw.copy()
    key, value = _pool(rng, N, Hkv, 1, D, torch.float16)
    key, value = key[:, :, 0, :].contiguous(), value[:, :, 0, :].contiguous()
    slots = rng.choice(NB * bs, size=N, replace=False).astype(np.int64)
    slots[3] = -1
    oracle.append(kw, vw, key, value, slots)
    rows_k, rows_v = _kv_rows(kw, Hkv, D), _kv_rows(vw, Hkv, D)
    rows_k0, rows_v0 = _kv_rows(k0, Hkv, D), _kv_rows(v0, Hkv, D)
    kk, vv = oracle.words(key), oracle.words(value)
    written = set()
    for i, s in enumerate(slots):
        if s < 0:
            continue
        written.add(int(s))
        assert np.array_equal(rows_k[:, s, :], kk[i]) and np.array_equal(rows_v[:, s, :], vv[i])
    for s in range(NB * bs):
        if s not in written:
            assert np.array_equal(rows_k[:, s], rows_k0[:, s])
            assert np.array_equal(rows_v[:, s], rows_v0[:, s])


def test_copy_blocks_round_trip_and_canaries():
    rng = np.random.default_rng(41)
    NB, Hkv, bs, D = 8, 2, 4, 8
    k, v = _pool(rng, NB, Hkv, bs, D, torch.bfloat16)
    kw, vw = oracle.words(k).copy(), oracle.words(v).copy()
    k0, v0 = kw.copy(), vw.copy()
    pairs = np.array([[1, 5], [1, 6], [2, 0]], dtype=np.int32)
    oracle.copy_blocks(kw, vw, pairs)
    for src, dst in pairs:
        assert np.array_equal(kw[dst], k0[src]) and np.array_equal(vw[dst], v0[src])
    for blk in range(NB):
        if blk not in pairs[:, 1]:
            assert np.array_equal(kw[blk], k0[blk]) and np.array_equal(vw[blk], v0[blk])


def test_bad_table_entry_is_reported():
    q, k, v, tables, lens, MB = _identity_case(seed=50, lens=(9, 9))
    bad = tables.copy()
    bad[0, 1] = k.shape[0]
    with pytest.raises(ValueError):
        oracle.paged_decode(q, k, v, bad, lens, 0.3)


def test_swap_round_trip_and_relation_to_copy_blocks():
    """Swapping blocks out and back into other blocks moves their bytes exactly as
    copy_blocks does; every other block is untouched."""
    rng = np.random.default_rng(42)
    NB, Hkv, bs, D = 9, 2, 4, 8
    k, v = _pool(rng, NB, Hkv, bs, D, torch.bfloat16)
    kw, vw = oracle.words(k).copy(), oracle.words(v).copy()
    k0, v0 = kw.copy(), vw.copy()
    out_ids, in_ids = [2, 7, 0], [5, 1, 8]
    hk = np.zeros((3, Hkv, bs, D), dtype=np.uint16)
    hv = np.zeros_like(hk)
    oracle.swap_blocks(kw, vw, hk, hv, out_ids, to_host=True)
    assert np.array_equal(kw, k0) and np.array_equal(vw, v0)          # reading changes nothing
    assert np.array_equal(hk, k0[out_ids]) and np.array_equal(hv, v0[out_ids])
    oracle.swap_blocks(kw, vw, hk, hv, in_ids, to_host=False)
    ck, cv = k0.copy(), v0.copy()
    oracle.copy_blocks(ck, cv, np.array(list(zip(out_ids, in_ids)), dtype=np.int32))
    assert np.array_equal(kw, ck) and np.array_equal(vw, cv)
    with pytest.raises(ValueError):
        oracle.swap_blocks(kw, vw, hk, hv, [NB], to_host=True)


# ------------------------------------------------------------ paged prefill

def _prefill_case(seed, lens, nq, H=4, Hkv=2, D=8, bs=4, dtype=torch.bfloat16):
    """Logical-order pool (as _identity_case) plus nq[b] query tokens per sequence."""
    q1, k, v, tables, lens, MB = _identity_case(seed, B=len(lens), H=H, Hkv=Hkv, D=D, bs=bs,
                                                lens=lens, dtype=dtype)
    rng = np.random.default_rng(seed + 1000)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = torch.from_numpy(rng.standard_normal((int(qs[-1]), H, D), dtype=np.float32)).to(dtype)
    return q, k, v, tables, lens, MB, qs


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("H,Hkv", [(4, 4), (8, 2)])
def test_prefill_whole_prompt_matches_sdpa_is_causal(dtype, H, Hkv):
    """A whole prompt (queries = every context token) is torch's causal SDPA,
    is_causal=True, over the logical slab, in float64."""
    lens = (37, 9, 1)
    q, k, v, tables, lens, MB, qs = _prefill_case(40 + H, lens, lens, H=H, Hkv=Hkv, dtype=dtype)
    out = oracle.paged_prefill(q, k, v, tables, lens, qs, 0.3)
    for b, L in enumerate(lens):
        Q = q[qs[b]:qs[b + 1]].to(torch.float64).permute(1, 0, 2)        # [H, L, D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            Q[None], _slab(k, b, MB, L)[None], _slab(v, b, MB, L)[None], scale=0.3,
            is_causal=True, enable_gqa=True)[0].permute(1, 0, 2)
        np.testing.assert_allclose(out[qs[b]:qs[b + 1]], ref.numpy(), rtol=RTOL, atol=1e-14)


def test_prefill_chunk_is_the_tail_of_the_whole_prompt():
    """Queries for the last n tokens give exactly the last n rows of the
    whole-prompt prefill with the same query vectors (chunked prefill)."""
    lens = (37, 22)
    q, k, v, tables, lens, MB, qs = _prefill_case(50, lens, lens)
    whole = oracle.paged_prefill(q, k, v, tables, lens, qs, 0.3)
    for n in (1, 5, 16):
        rows = np.concatenate([np.arange(qs[b + 1] - n, qs[b + 1]) for b in range(2)])
        qs_n = np.array([0, n, 2 * n], dtype=np.int32)
        part = oracle.paged_prefill(q[rows], k, v, tables, lens, qs_n, 0.3)
        assert np.array_equal(part, whole[rows])


def test_prefill_single_query_is_decode():
    lens = (37, 9)
    q, k, v, tables, lens, MB, qs = _prefill_case(51, lens, (1, 1))
    pre = oracle.paged_prefill(q, k, v, tables, lens, qs, 0.3)
    dec = oracle.paged_decode(q, k, v, tables, lens, 0.3)
    assert np.array_equal(pre, dec)


def test_prefill_closed_forms():
    """Position 0 sees only token 0 (out = V_0 exactly); a zero query weighs the
    causal prefix uniformly (out at position p = mean of V_0 .. V_p)."""
    lens = (23, 14)
    q, k, v, tables, lens, MB, qs = _prefill_case(52, lens, lens)
    out = oracle.paged_prefill(q, k, v, tables, lens, qs, 0.7)
    zero = oracle.paged_prefill(torch.zeros_like(q), k, v, tables, lens, qs, 0.7)
    for b, L in enumerate(lens):
        V = _slab(v, b, MB, L).numpy()                                  # [Hkv, L, D]
        for h in range(4):
            assert np.array_equal(out[qs[b], h], V[h // 2, 0])
            prefix_mean = np.cumsum(V[h // 2], axis=0) / np.arange(1, L + 1)[:, None]
            np.testing.assert_allclose(zero[qs[b]:qs[b + 1], h], prefix_mean, rtol=RTOL,
                                       atol=1e-14)


def test_prefill_block_permutation_invariance_is_bit_exact():
    lens = (29, 17)
    q, k, v, tables, lens, MB, qs = _prefill_case(53, lens, (11, 17))
    base = oracle.paged_prefill(q, k, v, tables, lens, qs, 0.35)
    perm = np.random.default_rng(3).permutation(k.shape[0])
    k2, v2 = torch.empty_like(k), torch.empty_like(v)
    k2[perm] = k
    v2[perm] = v
    moved = oracle.paged_prefill(q, k2, v2, perm[tables].astype(np.int32), lens, qs, 0.35)
    assert np.array_equal(base, moved)


def test_prefill_rejects_more_queries_than_context():
    q, k, v, tables, lens, MB, qs = _prefill_case(54, (5, 3), (5, 4))
    with pytest.raises(ValueError):
        oracle.paged_prefill(q, k, v, tables, lens, qs, 0.3)
