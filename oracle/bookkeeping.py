"""Naive model of PagedAttention's block bookkeeping -- oracle side.

TEST INFRASTRUCTURE ONLY: imported by tests/, the smoke check and the bench's
CPU-baseline leg, never by the library.  It shares no code with the library's
C++ block manager; the tests compare the two bit for bit.

What the pages fix, and where:

* the cache is cut into fixed-size blocks, each holding the keys and values of
  ``block_size`` tokens; a per-sequence block table maps logical block i to a
  physical block id ("PagedAttention" ops page, Concept -- What it is; "Paged
  Attention" KV-cache lesson, analogy table rows Unit and Mapping);
* a fresh block is taken from one global free pool only when the sequence's last
  block is full ("How it works -- The mechanics"; lesson: "allocate a new block
  only when decode fills the last one"), so the waste is at most one partly
  filled block per sequence;
* a finished sequence frees its blocks and they go back to the pool;
* sequences that share content point their tables at the same physical blocks,
  with a reference count, and a block is copied only when a sequence writes
  into it while it is shared (ops page, How it works and At a glance).

Readings where the pages are silent (fixed only so that two implementations
can be compared exactly; any order is correct by the pages):

* the free pool is a LIFO stack; it starts holding ``free_order`` with
  ``free_order[0]`` on top (default ``0, 1, 2, ...``);
* a freed sequence pushes its blocks in logical order, so its last block ends on
  top and is the next one handed out; shared blocks are only decremented;
* sequence ids count up from 0 and are never reused;
* ``reserve`` is all-or-nothing: if the pool cannot cover every block it needs
  (copy included) it changes nothing and reports exhaustion;
* ``cow(seq, i)`` gives the sequence a private copy of logical block i when the
  block is shared, and does nothing otherwise;
* a slot id is ``physical_block * block_size + offset``.

Preemption by swapping ("PagedAttention" ops page, How it works: when the free
pool empties the scheduler preempts a sequence and swaps its blocks to host
memory, then restores them later):

* ``swap_out(seq)`` returns the sequence's blocks in logical order (the caller
  copies them to host memory) and releases them exactly as ``free_seq`` would;
  the sequence keeps its length and holds no blocks while swapped;
* ``swap_in(seq)`` takes ``ceil(len / block_size)`` fresh blocks from the pool,
  all or nothing, and returns them in logical order (the caller copies the saved
  contents back into them); sharing is not restored: every block comes back
  private.

Prefix caching ("PagedAttention" glossary: the block table enables prefix
caching, where shared prompt prefixes across requests reuse already-computed KV
pages; ops page, Example: the shared system prompt is stored once and referenced
by every session's block table).  Readings:

* a full block's content is named by (the previous block of its sequence, or -1
  for the first block; the block's token ids), so a lookup walks the chain from
  the first block and a hit is exact -- no hashing;
* ``reserve_tokens(seq, tokens)`` is ``reserve`` that also records the token
  ids; when it fills a block whose predecessor is registered (or that is the
  sequence's first block), the block is registered unless that name is taken;
* ``new_cached(prompt)`` starts a sequence on the longest run of registered full
  blocks matching the prompt's full blocks (each shared, refcount + 1) and
  returns how many tokens that covers; a sequence whose token ids are unknown
  (created by ``new_seq`` and grown by ``reserve``) registers nothing;
* an entry lives only while its block is in use: when a block's count drops to
  0 (free, swap out, copy on write) its entry is dropped, and so is every entry
  chained below it (depth first, in registration order); blocks that come back
  by swap-in are not registered.
"""

from __future__ import annotations


class PoolExhausted(Exception):
    """The free pool cannot cover the request (the pages' trigger for preemption)."""


class BlockPoolModel:
    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = list(range(num_blocks)) if free_order is None else [int(x) for x in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the block ids")
        # The stack's top is the end of the list.
        self.free = list(reversed(order))
        self.refcount = [0] * self.num_blocks
        self.seqs = {}  # id -> {"blocks": [phys ids], "len": tokens, "swapped", "tokens"}
        self.next_id = 0
        self.cache = {}                     # (previous block or -1, token tuple) -> block
        self.key_of = {}                    # block -> its name in the cache
        self.children = {}                  # block -> names registered below it, in order

    # -- sequences -----------------------------------------------------------
    def new_seq(self) -> int:
        sid = self.next_id
        self.next_id += 1
        self.seqs[sid] = {"blocks": [], "len": 0, "swapped": False, "tokens": None}
        return sid

    def _resident(self, sid):
        seq = self.seqs[sid]
        if seq["swapped"]:
            raise ValueError(f"sequence {sid} is swapped out")
        return seq

    def fork(self, parent: int) -> int:
        """A new sequence that shares every block of ``parent`` (refcount + 1 each)."""
        src = self._resident(parent)
        sid = self.new_seq()
        self.seqs[sid]["blocks"] = list(src["blocks"])
        self.seqs[sid]["len"] = src["len"]
        self.seqs[sid]["tokens"] = None if src["tokens"] is None else list(src["tokens"])
        for b in src["blocks"]:
            self.refcount[b] += 1
        return sid

    def _pop(self) -> int:
        b = self.free.pop()
        self.refcount[b] = 1
        return b

    def reserve(self, sid: int, n_tokens: int):
        """Make room for ``n_tokens`` more tokens; return (slots, cow_pairs)."""
        seq = self._resident(sid)
        out = self._reserve(sid, n_tokens)      # all or nothing
        if n_tokens:
            seq["tokens"] = None                # token ids unknown from here on
        return out

    def reserve_tokens(self, sid: int, tokens):
        """``reserve`` for these token ids, registering every block it fills."""
        seq = self._resident(sid)
        known = seq["tokens"] is not None or seq["len"] == 0
        slots, pairs = self._reserve(sid, len(tokens))
        if not known:
            return slots, pairs
        if seq["tokens"] is None:
            seq["tokens"] = []
        start = len(seq["tokens"])
        seq["tokens"].extend(int(t) for t in tokens)
        bs = self.block_size
        # blocks that became full with this call, in logical order
        for i in range(start // bs, seq["len"] // bs):
            if (i + 1) * bs <= start:
                continue
            self._register(seq, i)
        return slots, pairs

    def _register(self, seq, i):
        blk = seq["blocks"][i]
        if blk in self.key_of:
            return
        prev = -1 if i == 0 else seq["blocks"][i - 1]
        if i > 0 and prev not in self.key_of:
            return
        key = (prev, tuple(seq["tokens"][i * self.block_size:(i + 1) * self.block_size]))
        if key in self.cache:
            return
        self.cache[key] = blk
        self.key_of[blk] = key
        if prev >= 0:
            self.children.setdefault(prev, []).append(key)

    def _drop(self, blk):
        key = self.key_of.pop(blk, None)
        if key is None:
            return
        del self.cache[key]
        if key[0] >= 0 and key in self.children.get(key[0], []):
            self.children[key[0]].remove(key)
        for child_key in list(self.children.pop(blk, [])):
            child = self.cache.get(child_key)
            if child is not None:
                self._drop(child)

    def new_cached(self, prompt):
        """A new sequence on the longest cached run of the prompt's full blocks;
        returns (sequence id, tokens covered)."""
        sid = self.new_seq()
        seq = self.seqs[sid]
        seq["tokens"] = []
        bs, prev = self.block_size, -1
        for i in range(len(prompt) // bs):
            chunk = tuple(int(t) for t in prompt[i * bs:(i + 1) * bs])
            blk = self.cache.get((prev, chunk))
            if blk is None:
                break
            self.refcount[blk] += 1
            seq["blocks"].append(blk)
            seq["tokens"].extend(chunk)
            prev = blk
        seq["len"] = len(seq["blocks"]) * bs
        return sid, seq["len"]

    def _reserve(self, sid: int, n_tokens: int):
        seq = self._resident(sid)
        bs = self.block_size
        length = seq["len"]
        # Count what the request needs before touching anything.
        need = 0
        pos = length
        for _ in range(n_tokens):
            if pos % bs == 0:
                need += 1
            pos += 1
        cow_needed = (n_tokens > 0 and length % bs != 0
                      and self.refcount[seq["blocks"][length // bs]] > 1)
        if cow_needed:
            need += 1
        if need > len(self.free):
            raise PoolExhausted(f"need {need} blocks, {len(self.free)} free")

        slots, pairs = [], []
        for _ in range(n_tokens):
            pos = seq["len"]
            if pos % bs == 0:
                # The last block is full (or there is none): take a fresh one.
                seq["blocks"].append(self._pop())
            else:
                cur = seq["blocks"][pos // bs]
                if self.refcount[cur] > 1:
                    # Writing into a shared block: copy it first.
                    fresh = self._pop()
                    self._decrement(cur)
                    seq["blocks"][pos // bs] = fresh
                    pairs.append((cur, fresh))
            slots.append(seq["blocks"][pos // bs] * bs + pos % bs)
            seq["len"] = pos + 1
        return slots, pairs

    def cow(self, sid: int, logical_block: int):
        """Give ``sid`` a private copy of one shared block; return the pair or None."""
        seq = self._resident(sid)
        cur = seq["blocks"][logical_block]
        if self.refcount[cur] <= 1:
            return None
        if not self.free:
            raise PoolExhausted("no free block for the copy")
        fresh = self._pop()
        self._decrement(cur)
        seq["blocks"][logical_block] = fresh  # the copy is not registered
        return (cur, fresh)

    def _decrement(self, b) -> None:
        """refcount - 1; at 0 the block leaves the cache and goes to the free pool."""
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self._drop(b)
            self.free.append(b)

    def _release(self, blocks) -> None:
        for b in blocks:
            self._decrement(b)

    def free_seq(self, sid: int) -> None:
        seq = self.seqs.pop(sid)
        self._release(seq["blocks"])

    def swap_out(self, sid: int):
        """Release the sequence's blocks to the pool; return them (logical order)."""
        seq = self._resident(sid)
        blocks = list(seq["blocks"])
        self._release(blocks)
        seq["blocks"] = []
        seq["swapped"] = True
        return blocks

    def swap_in(self, sid: int):
        """Give a swapped sequence fresh blocks for its whole length; return them."""
        seq = self.seqs[sid]
        if not seq["swapped"]:
            raise ValueError(f"sequence {sid} is not swapped out")
        need = -(-seq["len"] // self.block_size)
        if need > len(self.free):
            raise PoolExhausted(f"need {need} blocks, {len(self.free)} free")
        seq["blocks"] = [self._pop() for _ in range(need)]
        seq["swapped"] = False
        return list(seq["blocks"])

    # -- views ---------------------------------------------------------------
    def table(self, sid: int):
        return list(self.seqs[sid]["blocks"])

    def length(self, sid: int) -> int:
        return self.seqs[sid]["len"]

    def free_list(self):
        """Free ids from the top of the stack down (next to be handed out first)."""
        return list(reversed(self.free))

    def stats(self) -> dict:
        bs = self.block_size
        live = set()
        resident = [seq for seq in self.seqs.values() if not seq["swapped"]]
        for seq in resident:
            for t in range(seq["len"]):
                live.add((seq["blocks"][t // bs], t % bs))
        allocated = self.num_blocks - len(self.free)
        return {
            "free_blocks": len(self.free),
            "allocated_slots": allocated * bs,
            "live_slots": len(live),
            "live_tokens": sum(s["len"] for s in resident),
            "shared_blocks": sum(1 for r in self.refcount if r > 1),
            "num_seqs": len(resident),
            "swapped_seqs": len(self.seqs) - len(resident),
            "cached_blocks": len(self.cache),
        }


def contiguous_reservation_waste(lengths, reserve_tokens) -> dict:
    """The slab scheme the pages compare against: every request reserves a
    contiguous run of slots up front, sized for the longest output it might
    produce ("PagedAttention" ops page, Concept -- What it is; KV-cache lesson,
    problem statement and toy memory map).

    ``reserve_tokens`` is one reservation for every request, or a list with one
    per request.  A request can hold at most its reservation, so its live slots
    are min(length, reservation); the rest of the reservation is wasted."""
    n = len(lengths)
    if not hasattr(reserve_tokens, "__len__"):
        reserve = [int(reserve_tokens)] * n
    else:
        reserve = [int(r) for r in reserve_tokens]
        if len(reserve) != n:
            raise ValueError("one reservation per request")
    reserved = sum(reserve)
    live = sum(min(int(x), r) for x, r in zip(lengths, reserve))
    return {"reserved_slots": reserved, "live_slots": live, "wasted_slots": reserved - live}


def shared_prefix_groups(tables, lens, block_size: int, min_group_seqs: int = 2,
                         min_shared_blocks: int = 1, max_groups: int = 64):
    """Groups of consecutive sequences that share the leading blocks of their
    tables, for the shared-prefix decode (sequences forked from one prompt
    point their tables at the same blocks: "PagedAttention" ops page, At a
    glance and How it works).  Returns (group_start, group_shared_blocks) with
    len(group_start) == len(group_shared_blocks) + 1.

    The rule, taken from the batch order: a group starts at sequence i and
    takes i + 1, i + 2, ... as long as the leading table entries that all of
    them have in common with row i, counting only blocks full in every one of
    them, number at least ``min_shared_blocks``; it is kept when it has at
    least ``min_group_seqs`` sequences, otherwise the walk moves on to i + 1.
    Kept groups that are not back to back get a group sharing nothing between
    them; groups past ``max_groups`` entries are dropped."""
    n = len(lens)
    width = len(tables[0]) if n else 0

    def full(b):
        return min(max(int(lens[b]), 0) // block_size, width)

    kept = []
    i = 0
    while i < n and len(kept) < max_groups:
        common = full(i)
        j = i + 1
        while j < n:
            k = 0
            limit = min(common, full(j))
            while k < limit and tables[j][k] == tables[i][k]:
                k += 1
            if k < min_shared_blocks:
                break
            common = k
            j += 1
        if j - i >= min_group_seqs and common >= min_shared_blocks:
            kept.append((i, j, common))
            i = j
        else:
            i += 1
    starts, shared, end = [], [], 0
    for a, b, c in kept:
        gap = bool(shared) and a != end
        if len(shared) + (2 if gap else 1) > max_groups:
            break
        if gap:
            starts.append(end)
            shared.append(0)
        starts.append(a)
        shared.append(c)
        end = b
    starts.append(end)
    return starts, shared
