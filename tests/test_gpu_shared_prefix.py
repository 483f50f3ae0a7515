"""GPU parity of the shared-prefix decode (paged_attention_decode_shared_prefix)
against the CPU oracle, through the C ABI.

The shared-prefix decode computes the same attention as the plain decode (the
oracle's definition): the blocks that a group of sequences share are read once
per 128 query rows on the tensor cores and folded into each sequence's softmax
by log-sum-exp.  Every output element is compared with the float64 oracle at
|gpu - oracle| <= 2e-3 + 1e-2 |oracle|, on the full-size shared-prefix
workload after its copy-on-write step and on cases that mix groups of
different sizes and prefix lengths with ungrouped sequences, sequences whose
whole context is shared, and every supported (dtype, head_dim, block_size,
group size).  Block permutation must leave the output bit-identical.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_360_b200 as pkv
from paged_kv_cache_360_b200 import _lib
from paged_kv_cache_360_b200.workloads import make_workload, normal_tensor
from tests.gpu_helpers import compare, ensure_built, oracle_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


class Case:
    """A batch whose tables share leading blocks within groups.

    `spec` lists (num_seqs, shared_blocks, own_lens) per group in batch order;
    shared_blocks 0 makes the sequences ungrouped.  own_lens are the tokens
    each sequence has past the shared ones (0 = its whole context is shared)."""

    def __init__(self, spec, H, Hkv, D, bs, dtype, seed):
        rng = np.random.default_rng(seed)
        lens, rows, next_id = [], [], 0
        for n, shared, own in spec:
            prefix = list(range(next_id, next_id + shared))
            next_id += shared
            for k in range(n):
                L = shared * bs + int(own[k])
                mine = -(-int(own[k]) // bs)
                rows.append(prefix + list(range(next_id, next_id + mine)))
                next_id += mine
                lens.append(L)
        NB = next_id + 3
        perm = rng.permutation(NB).astype(np.int32)      # scatter the ids over the pool
        MB = max(1, max(len(r) for r in rows))
        self.tables = np.full((len(rows), MB), -1, dtype=np.int32)
        for i, r in enumerate(rows):
            self.tables[i, :len(r)] = perm[np.asarray(r, dtype=np.int64)]
        self.lens = np.asarray(lens, dtype=np.int32)
        self.B, self.H, self.Hkv, self.D, self.bs, self.dtype = len(rows), H, Hkv, D, bs, dtype
        self.scale = float(np.float32(1.0 / np.sqrt(D)))
        self.q = normal_tensor(rng, (self.B, H, D), dtype)
        self.k = normal_tensor(rng, (NB, Hkv, bs, D), dtype)
        self.v = normal_tensor(rng, (NB, Hkv, bs, D), dtype)
        starts, shared = [0], []
        for n, s, _ in spec:
            starts.append(starts[-1] + n)
            shared.append(s)
        self.group_start, self.group_shared = starts, shared

    # the oracle helpers read these attribute names
    @property
    def context_lens(self):
        return self.lens

    @property
    def block_tables(self):
        return self.tables

    @property
    def k_cache(self):
        return self.k

    @property
    def v_cache(self):
        return self.v

    @property
    def num_seqs(self):
        return self.B

    @property
    def num_heads(self):
        return self.H

    @property
    def head_dim(self):
        return self.D


def run_shared(case, group_start=None, group_shared=None, k=None, v=None, tables=None):
    dev = torch.device("cuda")
    q = case.q.to(dev)
    out = torch.full_like(q, float("nan"))
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pkv.paged_attention_decode_shared_prefix(
        out, q, (case.k if k is None else k).to(dev), (case.v if v is None else v).to(dev),
        torch.from_numpy(case.tables if tables is None else tables).to(dev),
        torch.from_numpy(case.lens).to(dev), case.scale,
        case.group_start if group_start is None else group_start,
        case.group_shared if group_shared is None else group_shared, err_flag=err)
    torch.cuda.synchronize()
    return out, int(err.item())


def run_plain(case):
    dev = torch.device("cuda")
    q = case.q.to(dev)
    out = torch.empty_like(q)
    pkv.paged_attention_decode(out, q, case.k.to(dev), case.v.to(dev),
                               torch.from_numpy(case.tables).to(dev),
                               torch.from_numpy(case.lens).to(dev), case.scale)
    torch.cuda.synchronize()
    return out


MIXED = [  # (sequences, shared blocks, own tokens per sequence)
    (3, 0, [5, 40, 1]),                            # ungrouped
    (40, 9, list(range(0, 400, 10))),              # more than one row tile at g <= 4
    (1, 4, [17]),                                  # a group of one
    (6, 1, [0, 1, 15, 16, 17, 300]),               # one shared block, an all-shared sequence
    (2, 0, [64, 3]),                               # ungrouped between groups
    (5, 25, [0, 0, 33, 128, 7]),                   # 25 shared blocks: several kv tiles
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("D,bs", [(128, 16), (64, 16), (128, 32), (64, 32)])
@pytest.mark.parametrize("group", [1, 4, 8, 16])
def test_mixed_groups_match_the_oracle(dtype, D, bs, group):
    case = Case(MIXED, H=2 * group, Hkv=2, D=D, bs=bs, dtype=dtype, seed=group * 7 + D + bs)
    out, err = run_shared(case)
    assert err == 0
    compare(out, oracle_decode(case), what=f"shared prefix mixed {str(dtype)[6:]} D={D} bs={bs} g={group}")


def test_two_tiles_per_item_and_a_partial_last_chunk():
    """Enough prefix work that an item takes two kv tiles (an odd number of
    tiles leaves a last item of one)."""
    spec = [(128, 64, [3 + (i % 50) for i in range(128)]), (64, 24, [1] * 64)]
    case = Case(spec, H=32, Hkv=8, D=128, bs=16, dtype=torch.bfloat16, seed=3)
    out, err = run_shared(case)
    assert err == 0
    compare(out, oracle_decode(case, threads=8), what="shared prefix two tiles per item")


def test_block_permutation_is_bit_identical():
    case = Case(MIXED, H=16, Hkv=4, D=128, bs=16, dtype=torch.bfloat16, seed=11)
    out, err = run_shared(case)
    NB = case.k.shape[0]
    perm = np.random.default_rng(5).permutation(NB)
    k2, v2 = torch.empty_like(case.k), torch.empty_like(case.v)
    k2[torch.from_numpy(perm)] = case.k
    v2[torch.from_numpy(perm)] = case.v
    t = case.tables.copy()
    t[t >= 0] = perm[t[t >= 0]]
    out2, err2 = run_shared(case, k=k2, v=v2, tables=t.astype(np.int32))
    assert err == 0 and err2 == 0
    assert torch.equal(out, out2)


def test_no_shared_blocks_equals_the_plain_decode_bit_for_bit():
    case = Case([(4, 0, [10, 300, 0, 77])], H=8, Hkv=2, D=128, bs=16, dtype=torch.bfloat16, seed=2)
    out, err = run_shared(case)
    assert err == 0
    assert torch.equal(out, run_plain(case))


def test_garbage_past_the_last_token_does_not_leak():
    spec = [(8, 3, [1, 5, 17, 40, 0, 2, 9, 100])]
    case = Case(spec, H=16, Hkv=4, D=128, bs=16, dtype=torch.float16, seed=13)
    for b in range(case.B):
        L = int(case.lens[b])
        if L % 16:
            blk = int(case.tables[b, L // 16])
            case.k[blk, :, L % 16:, :] = float("nan")
            case.v[blk, :, L % 16:, :] = float("inf")
    out, err = run_shared(case)
    assert err == 0 and torch.isfinite(out).all()
    compare(out, oracle_decode(case), what="shared prefix garbage tail")


def test_context_shorter_than_the_shared_blocks_is_flagged():
    case = Case([(3, 2, [4, 4, 4])], H=8, Hkv=2, D=128, bs=16, dtype=torch.bfloat16, seed=4)
    case.lens = case.lens.copy()
    case.lens[1] = 20   # < 2 shared blocks of 16 tokens
    _, err = run_shared(case)
    assert err & _lib.DEVERR_BAD_CONTEXT_LEN


def test_bad_group_arrays_are_rejected():
    case = Case([(3, 2, [4, 4, 4])], H=8, Hkv=2, D=128, bs=16, dtype=torch.bfloat16, seed=4)
    for gs, gb in (([0, 4], [2]), ([1, 1], [2]), ([0, 3], [99]), ([0, 3], [-1])):
        with pytest.raises(pkv.PkvError):
            run_shared(case, group_start=gs, group_shared=gb)
    odd = Case([(3, 2, [4, 4, 4])], H=6, Hkv=2, D=128, bs=16, dtype=torch.bfloat16, seed=4)
    with pytest.raises(pkv.PkvError) as e:
        run_shared(odd)
    assert e.value.status == 2


def _shared_prefix_step():
    """The shared-prefix workload after its copy-on-write and append step, built
    with the library's block manager; the groups come from the tables."""
    import bench
    wl = make_workload(3, seed=0)
    pairs, slots, tables, lens, key, value = bench.build_step(wl, bench.library_pool(pkv))
    k, v = wl.k_cache.clone(), wl.v_cache.clone()
    dev = torch.device("cuda")
    kd, vd = k.to(dev), v.to(dev)
    pkv.copy_blocks(kd, vd, torch.from_numpy(pairs).to(dev))
    pkv.paged_kv_append(kd, vd, key.to(dev), value.to(dev), torch.from_numpy(slots).to(dev))
    torch.cuda.synchronize()
    wl.k_cache, wl.v_cache = kd.cpu(), vd.cpu()
    wl.block_tables, wl.context_lens = tables, lens
    return wl


def test_full_size_shared_prefix_workload():
    """All 32 sequences of the shared-prefix workload: after the copy on write
    of the last prefix block, 63 blocks stay shared by every table."""
    wl = _shared_prefix_step()
    gs, gb = pkv.shared_prefix_groups(wl.block_tables, wl.context_lens, wl.block_size)
    assert list(gs) == [0, wl.num_seqs] and list(gb) == [wl.prefix_len // wl.block_size - 1]
    dev = torch.device("cuda")
    q, k, v = wl.q.to(dev), wl.k_cache.to(dev), wl.v_cache.to(dev)
    t, l = torch.from_numpy(wl.block_tables).to(dev), torch.from_numpy(wl.context_lens).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    pkv.paged_attention_decode_shared_prefix(out, q, k, v, t, l, wl.scale, gs, gb, err_flag=err)
    plain = torch.empty_like(q)
    pkv.paged_attention_decode(plain, q, k, v, t, l, wl.scale)
    torch.cuda.synchronize()
    assert err.item() == 0
    ref = oracle_decode(wl, threads=8)
    compare(out, ref, what="config 3 (shared-prefix-cow), shared-prefix decode")
    compare(plain, ref, what="config 3 (shared-prefix-cow), balanced")
