"""Replays a golden block-manager trace (tests/golden/*.txt) against a pool object.

The pool object needs: new_seq(), fork(sid), reserve(sid, n) -> (slots, pairs),
cow(sid, i), free_seq(sid), swap_out(sid) -> blocks, swap_in(sid) -> blocks,
table(sid), refcount(block) or .refcount[block], free_list(), stats() -> dict.  ``exhausted`` is the exception type the pool
raises when the free pool cannot cover a request.
"""

import os

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _ints(text):
    return [] if text == "-" else [int(x) for x in text.split(",")]


def _pairs(text):
    return [] if text == "-" else [tuple(int(y) for y in x.split(":")) for x in text.split(",")]


def _refcount(pool, block):
    rc = pool.refcount
    return rc(block) if callable(rc) else rc[block]


def play(name, factory, exhausted):
    path = os.path.join(GOLDEN, name)
    pool = None
    checked = 0
    for raw in open(path):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        lhs, _, rhs = line.partition("->")
        words, rhs = lhs.split(), rhs.strip()
        op = words[0]
        if op == "pool":
            pool = factory(int(words[1]), int(words[2]), _ints(words[3]))
            continue
        if op == "new":
            assert pool.new_seq() == int(rhs), line
        elif op == "fork":
            assert pool.fork(int(words[1])) == int(rhs), line
        elif op == "reserve":
            sid, n = int(words[1]), int(words[2])
            if rhs == "exhausted":
                before = (pool.table(sid), pool.free_list(), pool.stats())
                try:
                    pool.reserve(sid, n)
                except exhausted:
                    pass
                else:
                    raise AssertionError(f"expected exhaustion: {line}")
                assert (pool.table(sid), pool.free_list(), pool.stats()) == before, line
            else:
                slots, pairs = pool.reserve(sid, n)
                exp = rhs.split()
                assert exp[0] == "slots" and exp[2] == "pairs", line
                assert list(slots) == _ints(exp[1]), (line, slots)
                assert [tuple(p) for p in pairs] == _pairs(exp[3]), (line, pairs)
        elif op == "cow":
            pair = pool.cow(int(words[1]), int(words[2]))
            assert (None if pair is None else tuple(pair)) == \
                (None if rhs == "-" else _pairs(rhs)[0]), line
        elif op == "reserve_tokens":
            sid, toks = int(words[1]), [int(x) for x in words[2].split(":")]
            slots, pairs = pool.reserve_tokens(sid, toks)
            exp = rhs.split()
            assert list(slots) == _ints(exp[1]), (line, slots)
            assert [tuple(p) for p in pairs] == _pairs(exp[3]), (line, pairs)
        elif op == "new_cached":
            toks = [int(x) for x in words[1].split(":")]
            sid, covered = pool.new_cached(toks)
            exp = rhs.split()
            assert (sid, covered) == (int(exp[0]), int(exp[1])), (line, sid, covered)
        elif op in ("swap_out", "swap_in"):
            sid = int(words[1])
            fn = getattr(pool, op)
            if rhs == "exhausted":
                before = (pool.table(sid), pool.free_list(), pool.stats())
                try:
                    fn(sid)
                except exhausted:
                    pass
                else:
                    raise AssertionError(f"expected exhaustion: {line}")
                assert (pool.table(sid), pool.free_list(), pool.stats()) == before, line
            else:
                assert list(fn(sid)) == _ints(rhs), line
        elif op == "table":
            assert list(pool.table(int(words[1]))) == _ints(rhs), line
        elif op == "refcount":
            assert _refcount(pool, int(words[1])) == int(rhs), line
        elif op == "free":
            pool.free_seq(int(words[1]))
        elif op == "free_list":
            assert list(pool.free_list()) == _ints(rhs), line
        elif op == "stats":
            got = pool.stats()
            for item in rhs.split():
                key, val = item.split("=")
                assert got[key] == int(val), (line, got)
        else:
            raise ValueError(f"unknown op in {name}: {line}")
        checked += 1
    return checked
