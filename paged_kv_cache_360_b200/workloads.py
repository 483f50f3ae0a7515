"""Seeded synthetic inputs for paged decode attention.

This module only draws random numbers and lays out physical block ids.  It holds
none of the attention arithmetic and none of the block-manager rules; both the
CUDA path and the CPU oracle consume the buffers it returns, so it is the one
piece of code the two sides share.

Every draw comes from ``numpy.random.default_rng([seed, config, rank])`` (PCG64
seeded through SeedSequence), so a workload is a pure function of
``(config, seed, rank)``.  Floating-point values are drawn as float32 from
N(0, 1) and rounded to nearest-even into fp16 / bf16 by torch's dtype
conversion; the oracle widens those exact 16-bit values.

Workloads (shapes follow the pages' setting: a pool of fixed-size KV blocks, a
per-sequence block table that points into it, sequences of mixed length, and a
shared prompt prefix; sizes are those of a Llama-3-8B / 70B attention layer):

====  ============================  ======================================================
 id   name                          recipe
====  ============================  ======================================================
 1    tiny                          B 4, H = Hkv = 8, D 64, bs 16, fp16, L ~ U[1, 200],
                                    pool of 64 blocks in seeded random order
 2    llama3-8b-layer               B 64, H 32, Hkv 8, D 128, bs 16, bf16,
                                    L ~ U[128, 4096], NB = ceil(1.1 * sum(L) / bs)
 3    shared-prefix-cow             32 sequences, 1024-token shared prefix (64 blocks),
                                    suffix ~ U[0, 512] plus one new token, H 32, Hkv 8,
                                    D 128, bs 16, bf16
 4    long-context-split-k          B 8, L = 32768, H 32, Hkv 8, D 128, bs 16, bf16,
                                    NB = 16384 blocks in use + 1 % slack
 5    llama-70b-layer-mixed         B 256, H 64, Hkv 8, D 128, bs 32, bf16,
                                    L = clamp(round(exp(ln 600 + z)), 1, 8192), z ~ N(0,1),
                                    NB = ceil(used / 0.97) (about 3 % of ids stay free,
                                    interleaved with the used ones)
====  ============================  ======================================================

``context_lens`` are the lengths the decode step attends, the token appended in
the same step included: the appended token sits at position ``L - 1``.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

F16 = torch.float16
BF16 = torch.bfloat16

CONFIGS = {
    1: dict(name="tiny", B=4, H=8, Hkv=8, D=64, bs=16, dtype=F16),
    2: dict(name="llama3-8b-layer", B=64, H=32, Hkv=8, D=128, bs=16, dtype=BF16),
    3: dict(name="shared-prefix-cow", B=32, H=32, Hkv=8, D=128, bs=16, dtype=BF16,
            prefix=1024, suffix_max=512),
    4: dict(name="long-context-split-k", B=8, H=32, Hkv=8, D=128, bs=16, dtype=BF16,
            fixed_len=32768, partition_size=512),
    5: dict(name="llama-70b-layer-mixed", B=256, H=64, Hkv=8, D=128, bs=32, dtype=BF16),
}


@dataclass
class PagedWorkload:
    """One batch of synthetic decode inputs, all on the host.

    Attributes
    ----------
    k_cache, v_cache : ``[num_blocks, num_kv_heads, block_size, head_dim]``
        The whole pool, every slot filled with N(0, 1) values (they stand in
        for keys and values written by earlier steps).
    block_tables : int32 ``[num_seqs, max_blocks_per_seq]``
        Rows hold the physical ids of each sequence's blocks in logical order;
        entries past a sequence's last block are ``-1``.
    free_order : int32 ``[num_blocks]``
        A seeded permutation of all physical ids.  The block tables above take
        their ids from the front of it, in sequence order; an allocator seeded
        with it hands ids out in the same order.
    new_key, new_value : ``[num_new_tokens, num_kv_heads, head_dim]``
        Keys and values of the tokens appended in this step.
    """

    config: int
    name: str
    seed: int
    rank: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: torch.dtype
    scale: float
    context_lens: np.ndarray
    block_tables: np.ndarray
    free_order: np.ndarray
    q: torch.Tensor | None = None
    k_cache: torch.Tensor | None = None
    v_cache: torch.Tensor | None = None
    new_key: torch.Tensor | None = None
    new_value: torch.Tensor | None = None
    partition_size: int = 0
    # shared-prefix workload only
    prefix_len: int = 0
    suffix_lens: np.ndarray | None = None
    extra: dict = field(default_factory=dict)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def group(self) -> int:
        return self.num_heads // self.num_kv_heads

    def describe(self) -> dict:
        return dict(workload=self.name, config=self.config, seed=self.seed, rank=self.rank,
                    num_seqs=self.num_seqs, num_heads=self.num_heads,
                    num_kv_heads=self.num_kv_heads, head_dim=self.head_dim,
                    block_size=self.block_size, num_blocks=self.num_blocks,
                    dtype=str(self.dtype).replace("torch.", ""),
                    mean_context_len=float(np.mean(self.context_lens)) if self.num_seqs else 0.0,
                    max_context_len=int(np.max(self.context_lens)) if self.num_seqs else 0)


def rng_for(config: int, seed: int, rank: int = 0) -> np.random.Generator:
    return np.random.default_rng([int(seed), int(config), int(rank)])


def normal_tensor(rng: np.random.Generator, shape, dtype: torch.dtype,
                  chunk: int = 1 << 25) -> torch.Tensor:
    """N(0, 1) float32 draws rounded to ``dtype`` (round-to-nearest-even)."""
    out = torch.empty(shape, dtype=dtype)
    flat = out.view(-1)
    n = flat.numel()
    for start in range(0, n, chunk):
        stop = min(n, start + chunk)
        draw = rng.standard_normal(stop - start, dtype=np.float32)
        flat[start:stop] = torch.from_numpy(draw).to(dtype)
    return out


def _blocks_for(n_tokens: int, block_size: int) -> int:
    # Number of fixed-size blocks a run of n_tokens occupies (layout of the
    # synthetic tables only).
    return -(-int(n_tokens) // int(block_size))


def _tables_from_order(lens, order, block_size: int, max_blocks: int,
                       shared_prefix_ids=None) -> np.ndarray:
    """Give each sequence the next ids of ``order``; shared ids go first."""
    B = len(lens)
    tables = np.full((B, max(1, max_blocks)), -1, dtype=np.int32)
    cursor = 0
    n_shared = 0 if shared_prefix_ids is None else len(shared_prefix_ids)
    for b in range(B):
        nb = _blocks_for(lens[b], block_size)
        if n_shared:
            tables[b, :n_shared] = shared_prefix_ids
        own = nb - n_shared
        tables[b, n_shared:n_shared + own] = order[cursor:cursor + own]
        cursor += own
    return tables


def make_workload(config: int, seed: int = 0, rank: int = 0, materialize: bool = True,
                  num_seqs: int | None = None) -> PagedWorkload:
    """Build the synthetic batch of one workload.

    ``num_seqs`` overrides the batch size (smaller parity cases); everything
    else keeps the recipe.  ``materialize=False`` skips the value tensors.
    """
    cfg = CONFIGS[config]
    rng = rng_for(config, seed, rank)
    B = cfg["B"] if num_seqs is None else int(num_seqs)
    bs, D, H, Hkv, dtype = cfg["bs"], cfg["D"], cfg["H"], cfg["Hkv"], cfg["dtype"]
    prefix_len = 0
    suffix_lens = None

    if config == 1:
        lens = rng.integers(1, 200, size=B, endpoint=True)
        num_blocks = 64 if B <= 4 else max(64, sum(_blocks_for(x, bs) for x in lens))
    elif config == 2:
        lens = rng.integers(128, 4096, size=B, endpoint=True)
        num_blocks = math.ceil(1.1 * int(lens.sum()) / bs)
    elif config == 3:
        prefix_len = cfg["prefix"]
        suffix_lens = rng.integers(0, cfg["suffix_max"], size=B, endpoint=True)
        lens = prefix_len + suffix_lens + 1
        n_prefix = _blocks_for(prefix_len, bs)
        own = sum(_blocks_for(x, bs) - n_prefix for x in lens)
        # room for the shared prefix, each sequence's own blocks, one private
        # copy of a prefix block per sequence, and 10 % slack
        num_blocks = math.ceil(1.1 * (n_prefix + own + B))
    elif config == 4:
        lens = np.full(B, cfg["fixed_len"], dtype=np.int64)
        used = sum(_blocks_for(x, bs) for x in lens)
        num_blocks = used + math.ceil(0.01 * used)
    elif config == 5:
        z = rng.standard_normal(B)
        lens = np.clip(np.rint(np.exp(math.log(600.0) + 1.0 * z)), 1, 8192).astype(np.int64)
        used = sum(_blocks_for(x, bs) for x in lens)
        num_blocks = math.ceil(used / 0.97)
    else:
        raise ValueError(f"unknown workload {config}")

    lens = np.asarray(lens, dtype=np.int64)
    order = rng.permutation(num_blocks).astype(np.int32)
    max_blocks = max(_blocks_for(x, bs) for x in lens) if B else 1
    if config == 3:
        n_prefix = _blocks_for(prefix_len, bs)
        prefix_ids = order[:n_prefix]
        tables = _tables_from_order(lens, order[n_prefix:], bs, max_blocks, prefix_ids)
    else:
        tables = _tables_from_order(lens, order, bs, max_blocks)

    wl = PagedWorkload(
        config=config, name=cfg["name"], seed=seed, rank=rank, num_seqs=B, num_heads=H,
        num_kv_heads=Hkv, head_dim=D, block_size=bs, num_blocks=int(num_blocks), dtype=dtype,
        scale=float(np.float32(1.0 / math.sqrt(D))),
        context_lens=lens.astype(np.int32), block_tables=tables, free_order=order,
        partition_size=cfg.get("partition_size", 0), prefix_len=prefix_len,
        suffix_lens=None if suffix_lens is None else suffix_lens.astype(np.int32))
    if materialize:
        wl.q = normal_tensor(rng, (B, H, D), dtype)
        wl.k_cache = normal_tensor(rng, (num_blocks, Hkv, bs, D), dtype)
        wl.v_cache = normal_tensor(rng, (num_blocks, Hkv, bs, D), dtype)
        n_new = int((suffix_lens + 1).sum()) if config == 3 else B
        wl.new_key = normal_tensor(rng, (n_new, Hkv, D), dtype)
        wl.new_value = normal_tensor(rng, (n_new, Hkv, D), dtype)
    return wl


def custom_workload(*, num_seqs, num_heads, num_kv_heads, head_dim, block_size, context_lens,
                    dtype=BF16, seed=0, slack_blocks=3, max_blocks_per_seq=None,
                    shuffle=True, value_scale=1.0) -> PagedWorkload:
    """A workload with explicit lengths (edge cases: empty, one token, ragged tails)."""
    rng = np.random.default_rng([int(seed), 99, len(context_lens)])
    lens = np.asarray(context_lens, dtype=np.int64)
    used = sum(_blocks_for(x, block_size) for x in lens)
    num_blocks = max(1, used + int(slack_blocks))
    order = rng.permutation(num_blocks).astype(np.int32) if shuffle else \
        np.arange(num_blocks, dtype=np.int32)
    max_blocks = max([_blocks_for(x, block_size) for x in lens] + [1])
    if max_blocks_per_seq is not None:
        max_blocks = max(max_blocks, int(max_blocks_per_seq))
    tables = _tables_from_order(lens, order, block_size, max_blocks)
    wl = PagedWorkload(
        config=0, name="custom", seed=seed, rank=0, num_seqs=len(lens), num_heads=num_heads,
        num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size,
        num_blocks=num_blocks, dtype=dtype, scale=float(np.float32(1.0 / math.sqrt(head_dim))),
        context_lens=lens.astype(np.int32), block_tables=tables, free_order=order)
    wl.q = normal_tensor(rng, (len(lens), num_heads, head_dim), dtype)
    wl.k_cache = normal_tensor(rng, (num_blocks, num_kv_heads, block_size, head_dim), dtype)
    wl.v_cache = normal_tensor(rng, (num_blocks, num_kv_heads, block_size, head_dim), dtype)
    if value_scale != 1.0:
        wl.q = (wl.q.float() * value_scale).to(dtype)
    wl.new_key = normal_tensor(rng, (len(lens), num_kv_heads, head_dim), dtype)
    wl.new_value = normal_tensor(rng, (len(lens), num_kv_heads, head_dim), dtype)
    return wl


def random_slot_mapping(rng: np.random.Generator, num_slots: int, n: int,
                        pad_every: int = 0) -> np.ndarray:
    """``n`` distinct slot ids in ``[0, num_slots)``; every ``pad_every``-th is -1."""
    slots = rng.choice(num_slots, size=n, replace=False).astype(np.int64)
    if pad_every:
        slots[pad_every - 1::pad_every] = -1
    return slots


def random_block_pairs(rng: np.random.Generator, num_blocks: int, m: int) -> np.ndarray:
    """``m`` (src, dst) pairs: distinct destinations, no destination is a source."""
    ids = rng.permutation(num_blocks)
    dst = ids[:m]
    src = rng.choice(ids[m:], size=m, replace=True) if m else ids[:0]
    return np.stack([src, dst], axis=1).astype(np.int32)


def shard_seed(seed: int, rank: int) -> tuple[int, int]:
    """Each rank of a multi-GPU run draws its own batch: (seed, rank) keys the draw."""
    return int(seed), int(rank)


# ------------------------------------------------------------------ prefill

PREFILL_CONFIGS = {
    # 16 requests of a Llama-3-8B layer: half are whole prompts, half a 512-token
    # chunk at the end of a longer context (chunked prefill)
    "prefill-llama3-8b-layer": dict(B=16, H=32, Hkv=8, D=128, bs=16, dtype=BF16, lo=512,
                                    hi=4096, chunk=512),
    # small case for the oracle
    "prefill-tiny": dict(B=4, H=8, Hkv=2, D=128, bs=16, dtype=BF16, lo=1, hi=300, chunk=64),
}


@dataclass
class PrefillWorkload:
    """One batch of prefill inputs on the host.

    Sequence b holds ``context_lens[b]`` tokens; its last ``n_b =
    query_start[b+1] - query_start[b]`` are the step's query tokens, whose keys
    and values are rows ``query_start[b] ..`` of ``new_key`` / ``new_value``.
    The earlier tokens' keys and values are whatever the pool holds.  Block ids
    are handed out by a block manager seeded with ``free_order``."""

    name: str
    seed: int
    rank: int
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    dtype: torch.dtype
    scale: float
    context_lens: np.ndarray
    query_start: np.ndarray
    free_order: np.ndarray
    q: torch.Tensor | None = None
    k_cache: torch.Tensor | None = None
    v_cache: torch.Tensor | None = None
    new_key: torch.Tensor | None = None
    new_value: torch.Tensor | None = None

    @property
    def num_tokens(self) -> int:
        return int(self.query_start[-1])


def make_prefill_workload(name: str = "prefill-llama3-8b-layer", seed: int = 0, rank: int = 0,
                          materialize: bool = True) -> PrefillWorkload:
    """Lengths L ~ U[lo, hi]; even-indexed requests query their whole prompt,
    odd-indexed ones the last min(chunk, L) tokens.  The pool has 3 % more
    blocks than the contexts fill, ids in a seeded random order."""
    c = PREFILL_CONFIGS[name]
    rng = np.random.default_rng([int(seed), 1000 + list(PREFILL_CONFIGS).index(name), int(rank)])
    B, bs = c["B"], c["bs"]
    lens = rng.integers(c["lo"], c["hi"] + 1, size=B).astype(np.int32)
    nq = np.where(np.arange(B) % 2 == 0, lens, np.minimum(lens, c["chunk"])).astype(np.int32)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    used = int(sum(_blocks_for(x, bs) for x in lens))
    num_blocks = int(math.ceil(used * 1.03)) + 1
    wl = PrefillWorkload(
        name=name, seed=seed, rank=rank, num_seqs=B, num_heads=c["H"], num_kv_heads=c["Hkv"],
        head_dim=c["D"], block_size=bs, num_blocks=num_blocks, dtype=c["dtype"],
        scale=float(np.float32(1.0 / math.sqrt(c["D"]))), context_lens=lens, query_start=qs,
        free_order=rng.permutation(num_blocks).astype(np.int32))
    if materialize:
        T = int(qs[-1])
        wl.q = normal_tensor(rng, (T, c["H"], c["D"]), c["dtype"])
        wl.k_cache = normal_tensor(rng, (num_blocks, c["Hkv"], bs, c["D"]), c["dtype"])
        wl.v_cache = normal_tensor(rng, (num_blocks, c["Hkv"], bs, c["D"]), c["dtype"])
        wl.new_key = normal_tensor(rng, (T, c["Hkv"], c["D"]), c["dtype"])
        wl.new_value = normal_tensor(rng, (T, c["Hkv"], c["D"]), c["dtype"])
    return wl
