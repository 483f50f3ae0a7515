"""GPU parity of the tcgen05 paged prefill against the CPU oracle, through the C ABI.

Every output row within |gpu - oracle| <= 2e-3 + 1e-2 |oracle| of the float64
oracle on cases that span several 128-row query tiles and 128-token kv tiles
with ragged tails: whole prompts, chunks of prompts (queries = the last n
tokens), single decode tokens, sequences with no queries, every group size the
kernel packs, both head sizes and block sizes.  Garbage past the context must
not reach the output; block permutation leaves it bit-identical; bad table
entries and query counts are flagged, not faulted on.  A Llama-3-8B-shaped
batch is checked on sampled rows (a row at position p is decode over the
first p + 1 tokens, computed by the oracle one by one).
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_360_b200 as pkv
from paged_kv_cache_360_b200.workloads import custom_workload, normal_tensor
from tests.gpu_helpers import compare, ensure_built, prefix_rows, words

pytestmark = pytest.mark.gpu

DTYPES = [torch.bfloat16, torch.float16]


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


def _case(lens, nq, H, Hkv, D, bs, dtype, seed):
    wl = custom_workload(num_seqs=len(lens), num_heads=H, num_kv_heads=Hkv, head_dim=D,
                         block_size=bs, context_lens=lens, dtype=dtype, seed=seed)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    rng = np.random.default_rng([seed, 5])
    q = normal_tensor(rng, (int(qs[-1]), H, D), dtype)
    return wl, q, qs


def _run(wl, q, qs, k=None, v=None, tables=None, err=None):
    out = torch.zeros(q.shape, dtype=q.dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda") if err is None else err
    t = wl.block_tables if tables is None else tables
    pkv.paged_attention_prefill(
        out, q.cuda(), (wl.k_cache if k is None else k).cuda(), (wl.v_cache if v is None else v).cuda(),
        torch.from_numpy(np.ascontiguousarray(t)).cuda(),
        torch.from_numpy(np.ascontiguousarray(wl.context_lens)).cuda(),
        torch.from_numpy(qs).cuda(), wl.scale, err_flag=err)
    torch.cuda.synchronize()
    return out, int(err.item())


def _ref(wl, q, qs, k=None, v=None):
    return oracle.paged_prefill(q, wl.k_cache if k is None else k, wl.v_cache if v is None else v,
                                wl.block_tables, wl.context_lens, qs, wl.scale)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("D,bs", [(128, 16), (128, 32), (64, 16)])
@pytest.mark.parametrize("group", [1, 4, 8])
def test_prefill_whole_prompts(dtype, D, bs, group):
    lens = [1, 17, 128, 129, 300]
    wl, q, qs = _case(lens, lens, group * 2, 2, D, bs, dtype, seed=group + D)
    out, err = _run(wl, q, qs)
    assert err == 0
    compare(out, _ref(wl, q, qs), what=f"whole prompts g={group} D={D} bs={bs}")


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("group", [2, 16])
def test_prefill_chunks_decode_rows_and_empty(dtype, group):
    """Chunks of prompts (queries = the last n tokens), decode rows, no queries."""
    lens = [300, 77, 513, 40, 260, 9]
    nq = [64, 77, 5, 1, 0, 9]
    wl, q, qs = _case(lens, nq, group * 2, 2, 128, 16, dtype, seed=7 * group)
    out, err = _run(wl, q, qs)
    assert err == 0
    compare(out, _ref(wl, q, qs), what=f"chunks g={group}")


def test_prefill_writes_only_the_query_rows():
    """Output rows past the last sequence's queries keep what they held, and
    every written row matches the oracle, for tiles that leave as one bulk
    store (whole 32-token tiles at g = 4) and ragged last tiles alike."""
    lens, nq = [300, 64, 129, 37], [96, 64, 33, 37]
    wl, q, qs = _case(lens, nq, 16, 4, 128, 16, torch.bfloat16, seed=53)
    extra = 40
    q_all = torch.cat([q, normal_tensor(np.random.default_rng(54), (extra, 16, 128), torch.bfloat16)])
    out = torch.full(q_all.shape, float("nan"), dtype=q_all.dtype, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    pkv.paged_attention_prefill(
        out, q_all.cuda(), wl.k_cache.cuda(), wl.v_cache.cuda(),
        torch.from_numpy(np.ascontiguousarray(wl.block_tables)).cuda(),
        torch.from_numpy(np.ascontiguousarray(wl.context_lens)).cuda(),
        torch.from_numpy(qs).cuda(), wl.scale, err_flag=err)
    torch.cuda.synchronize()
    assert err.item() == 0
    n = int(qs[-1])
    assert torch.isnan(out[n:].float()).all()
    compare(out[:n], _ref(wl, q, qs), what="prefill rows of the call")


def test_prefill_ignores_garbage_past_the_context():
    lens = [3, 17, 140, 250]
    wl, q, qs = _case(lens, lens, 8, 2, 128, 16, torch.bfloat16, seed=31)
    ref = _ref(wl, q, qs)
    for b, L in enumerate(lens):
        blk = int(wl.block_tables[b, (L - 1) // 16])
        wl.k_cache[blk, :, L % 16 or 16:, :] = float("nan")
        wl.v_cache[blk, :, L % 16 or 16:, :] = float("inf")
    out, err = _run(wl, q, qs)
    assert err == 0 and torch.isfinite(out).all()
    compare(out, ref, what="garbage tail")


def test_prefill_block_permutation_is_bit_identical():
    lens = [200, 131]
    wl, q, qs = _case(lens, [150, 131], 16, 4, 128, 16, torch.bfloat16, seed=41)
    base, _ = _run(wl, q, qs)
    perm = np.random.default_rng(3).permutation(wl.num_blocks)
    k2, v2 = torch.empty_like(wl.k_cache), torch.empty_like(wl.v_cache)
    k2[perm] = wl.k_cache
    v2[perm] = wl.v_cache
    tables = np.where(wl.block_tables >= 0, perm[np.maximum(wl.block_tables, 0)], -1).astype(np.int32)
    moved, _ = _run(wl, q, qs, k=k2, v=v2, tables=tables)
    assert torch.equal(base, moved)


def test_prefill_is_deterministic():
    lens = [384, 100]
    wl, q, qs = _case(lens, lens, 32, 8, 128, 16, torch.bfloat16, seed=43)
    a, _ = _run(wl, q, qs)
    b, _ = _run(wl, q, qs)
    assert torch.equal(a, b)


def test_prefill_flags_bad_table_entries_and_query_counts():
    lens = [40, 20]
    wl, q, qs = _case(lens, lens, 8, 2, 128, 16, torch.float16, seed=47)
    tables = wl.block_tables.copy()
    tables[0, 1] = wl.num_blocks + 5
    _, err = _run(wl, q, qs, tables=tables)
    assert err & 1
    bad = qs.copy()
    bad[1] = 50                                    # sequence 0 claims 50 queries for 40 tokens
    _, err = _run(wl, q, bad)
    assert err & 32


def test_prefill_rejects_bad_arguments():
    lens = [10]
    wl, q, qs = _case(lens, lens, 12, 4, 128, 16, torch.bfloat16, seed=53)   # group 3
    with pytest.raises(pkv.PkvError):
        _run(wl, q, qs)
    wl, q, qs = _case(lens, lens, 8, 2, 128, 16, torch.bfloat16, seed=53)
    out = torch.zeros(q.shape, dtype=q.dtype, device="cuda")
    with pytest.raises(pkv.PkvError):           # host tensors
        pkv.paged_attention_prefill(out, q, wl.k_cache, wl.v_cache, torch.from_numpy(wl.block_tables),
                                    torch.from_numpy(wl.context_lens), torch.from_numpy(qs), wl.scale)


def test_prefill_llama3_8b_layer_sampled():
    """8 prompts of 1024-2048 tokens (one a 512-token chunk of a 2048-token
    context), H 32, Hkv 8, D 128, bs 16, bf16: 256 sampled (row, head) outputs."""
    lens = [2048, 1536, 1024, 2047, 1300, 2048, 1111, 1900]
    nq = list(lens)
    nq[5] = 512
    wl, q, qs = _case(lens, nq, 32, 8, 128, 16, torch.bfloat16, seed=61)
    out, err = _run(wl, q, qs)
    assert err == 0
    rng = np.random.default_rng(5)
    g = out.float().cpu().double().numpy()
    for _ in range(64):
        b = int(rng.integers(0, len(lens)))
        if nq[b] == 0:
            continue
        i = int(rng.integers(0, nq[b]))
        row = int(qs[b]) + i
        pos = lens[b] - nq[b] + i
        # decode over the first pos + 1 tokens with this query row
        ref = oracle.paged_decode(q[row:row + 1], wl.k_cache, wl.v_cache, wl.block_tables[b:b + 1],
                                  np.array([pos + 1], dtype=np.int32), wl.scale)[0]
        compare(out[row:row + 1], ref[None], what=f"sampled b={b} pos={pos}")


@pytest.mark.parametrize("dtype", DTYPES)
def test_prefix_cached_request_prefills_only_its_own_tokens(dtype):
    """Block manager, prefix cache and chunked prefill together: request B shares
    request A's system prompt, starts on A's cached full blocks, appends and
    prefills only its own tokens (a chunk at the end of its context); every
    query row of both requests matches the oracle's prefill over the whole
    context, read from the oracle's own copy of the pool."""
    bs, Hkv, H, D, NB = 16, 2, 8, 128, 64
    rng = np.random.default_rng(71)
    system = list(rng.integers(0, 1000, size=70))
    prompts = [system + list(rng.integers(0, 1000, size=m)) for m in (30, 45)]
    pool = pkv.Pool(NB, bs, rng.permutation(NB))
    model = oracle.BlockPoolModel(NB, bs, pool.free_list())
    k0 = normal_tensor(rng, (NB, Hkv, bs, D), dtype)
    v0 = normal_tensor(rng, (NB, Hkv, bs, D), dtype)
    kd, vd = k0.cuda(), v0.cuda()
    kw, vw = words(k0).copy(), words(v0).copy()
    scale = float(np.float32(1.0 / np.sqrt(D)))
    covered_all = []
    for prompt in prompts:
        sid, covered = pool.new_cached(prompt)
        assert (sid, covered) == model.new_cached(prompt)
        slots, pairs = pool.reserve_tokens(sid, prompt[covered:])
        assert (list(slots), pairs) == model.reserve_tokens(sid, prompt[covered:])
        kr, vr = prefix_rows(prompt, Hkv, D, dtype)
        pkv.paged_kv_append(kd, vd, kr[covered:].cuda(), vr[covered:].cuda(), torch.from_numpy(slots).cuda())
        oracle.append(kw, vw, kr[covered:], vr[covered:], slots)
        n = len(prompt) - covered
        q = normal_tensor(rng, (n, H, D), dtype)
        table = np.array([pool.table(sid)], dtype=np.int32)
        lens = np.array([len(prompt)], dtype=np.int32)
        qs = np.array([0, n], dtype=np.int32)
        out = torch.zeros((n, H, D), dtype=dtype, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        pkv.paged_attention_prefill(out, q.cuda(), kd, vd, torch.from_numpy(table).cuda(),
                                    torch.from_numpy(lens).cuda(), torch.from_numpy(qs).cuda(), scale,
                                    err_flag=err)
        torch.cuda.synchronize()
        assert err.item() == 0
        k_or = torch.from_numpy(kw.view(np.int16)).view(dtype).reshape(k0.shape)
        v_or = torch.from_numpy(vw.view(np.int16)).view(dtype).reshape(v0.shape)
        compare(out, oracle.paged_prefill(q, k_or, v_or, table, lens, qs, scale),
                what=f"prefix-cached prefill, {covered} cached tokens")
        covered_all.append(covered)
    assert covered_all == [0, 64]              # four full 16-token blocks of the system prompt
    assert np.array_equal(words(kd.cpu()), kw) and np.array_equal(words(vd.cpu()), vw)


def _sampled_rows(out, wl, q, qs, lens, nq, rng, count):
    for _ in range(count):
        b = int(rng.integers(0, len(lens)))
        if nq[b] == 0:
            continue
        i = int(rng.integers(0, nq[b]))
        row = int(qs[b]) + i
        pos = int(lens[b]) - int(nq[b]) + i
        ref = oracle.paged_decode(q[row:row + 1], wl.k_cache, wl.v_cache, wl.block_tables[b:b + 1],
                                  np.array([pos + 1], dtype=np.int32), wl.scale)[0]
        compare(out[row:row + 1], ref[None], what=f"sampled b={b} pos={pos}")


def test_prefill_long_context_chunk_sampled():
    """A 256-token chunk at the end of a 32k-token context (256 kv tiles, the
    block table fetched in 64 chunks of 32 entries) next to a short prompt."""
    lens, nq = [32768, 300], [256, 300]
    wl, q, qs = _case(lens, nq, 32, 8, 128, 16, torch.bfloat16, seed=81)
    out, err = _run(wl, q, qs)
    assert err == 0
    _sampled_rows(out, wl, q, qs, lens, nq, np.random.default_rng(6), 24)
    # the chunk's last row is the full causal row over all 32768 tokens
    row = int(qs[1]) - 1
    ref = oracle.paged_decode(q[row:row + 1], wl.k_cache, wl.v_cache, wl.block_tables[0:1],
                              np.array([32768], dtype=np.int32), wl.scale)[0]
    compare(out[row:row + 1], ref[None], what="last row of the 32k context")


def test_prefill_multi_head_full_size_sampled():
    """g = 1 (every query head has its own kv head): 128 query tokens per tile."""
    lens = [1536, 777, 2048, 40]
    wl, q, qs = _case(lens, lens, 16, 16, 128, 32, torch.float16, seed=83)
    out, err = _run(wl, q, qs)
    assert err == 0
    _sampled_rows(out, wl, q, qs, lens, lens, np.random.default_rng(7), 24)
