"""The oracle's pins must reject plausible mistakes (no GPU).

Each mutant below is a copy of oracle/pkv_oracle.c (or, for WASTE_MUTANTS, of
the bookkeeping model's slab-waste function) with one deliberate
mistake -- a wrong index, a dropped term, a wrong sign, a transposed operand, a
wrong constant.  It is compiled on the CPU and test_oracle_pins.py is run
against it in a child process (PKV_ORACLE_LIB points the oracle at the
mutant); every mutant has to make that run fail.  A crash of the child counts
as a failure too.  The mutants live only in a temporary directory.
"""

import concurrent.futures
import os
import subprocess
import sys
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pkv_oracle.c")

MUTANTS = {
    "block index uses modulo": ("table_row[t / block_size]", "table_row[t % block_size]"),
    "offset and block swapped": ("int64_t off = t % block_size;",
                                 "int64_t off = (t / block_size) % block_size;"),
    "pool layout heads/offset transposed":
        ("(((int64_t)phys * num_kv_heads + hk) * block_size + off) * D",
         "(((int64_t)phys * block_size + off) * num_kv_heads + hk) * D"),
    "scale dropped": ("scores[t] = scale * dot;", "scores[t] = dot;"),
    "softmax exponent sign": ("double e = exp(scores[t] - m);", "double e = exp(m - scores[t]);"),
    "normalisation dropped": ("for (int32_t d = 0; d < D; ++d) out[d] /= l;", ""),
    "query/key operand transposed": ("dot += q[d] * K[t * D + d];",
                                     "dot += q[d] * K[d * D + (t % D)];"),
    "values read from keys": ("out[d] += scores[t] * V[t * D + d];",
                              "out[d] += scores[t] * K[t * D + d];"),
    "first value term dropped": ("for (int64_t t = 0; t < L; ++t)\n        for (int32_t d = 0; d < D; ++d) out[d] +=",
                                 "for (int64_t t = 1; t < L; ++t)\n        for (int32_t d = 0; d < D; ++d) out[d] +="),
    "GQA mapping interleaved": ("for (int32_t h = hk * group; h < (hk + 1) * group; ++h)",
                                "for (int32_t h = hk; h < H; h += Hkv)"),
    "fp16 exponent bias": ("exp - 25", "exp - 24"),
    "fp16 subnormal scale": ("ldexp((double)frac, -24)", "ldexp((double)frac, -25)"),
    "bf16 shift": ("(uint32_t)b << 16", "(uint32_t)b << 15"),
    "dtype dispatch inverted": ("return dtype == ORACLE_BF16 ?", "return dtype != ORACLE_BF16 ?"),
    "split merge weight dropped": ("denom += w * lp[p];", "denom += lp[p];"),
    "split partition drops a token": ("int64_t t0 = p * P, t1 = (p + 1) * P < L ? (p + 1) * P : L;",
                                      "int64_t t0 = p * P, t1 = (p + 1) * P < L ? (p + 1) * P - 1 : L;"),
    "append offset": ("int64_t phys = slot / block_size, off = slot % block_size;",
                      "int64_t phys = slot % block_size, off = slot / block_size;"),
    "append skips value": ("memcpy(v_cache + dst, value + src, sizeof(uint16_t) * (size_t)D);", ""),
    "copy skips value": ("memcpy(v_cache + dst * block_words, v_cache + src * block_words,\n"
                         "               sizeof(uint16_t) * (size_t)block_words);", ""),
    "copy direction reversed": ("memcpy(k_cache + dst * block_words, k_cache + src * block_words,",
                                "memcpy(k_cache + src * block_words, k_cache + dst * block_words,"),
    "swap uses the list position as the block": ("uint16_t* pk = k_cache + blk * block_words;",
                                                 "uint16_t* pk = k_cache + i * block_words;"),
    "prefill causal bound off by one": ("oracle_attend_dense(qd, K, V, p + 1, D,",
                                        "oracle_attend_dense(qd, K, V, p, D,"),
    "prefill sees the whole context": ("oracle_attend_dense(qd, K, V, p + 1, D,",
                                       "oracle_attend_dense(qd, K, V, L, D,"),
    "prefill position ignores the context": ("int64_t p = L - n + i;", "int64_t p = i;"),
    "prefill query row ignores the sequence offset": ("int64_t row = query_start[b] + i;",
                                                      "int64_t row = i;"),
    "prefill GQA mapping interleaved": ("int32_t h = hk * group + j;", "int32_t h = hk + j * Hkv;"),
    "swap direction inverted": ("        if (to_host) {\n            memcpy(hk, pk,",
                                "        if (!to_host) {\n            memcpy(hk, pk,"),
    "listed sequence index not checked": ("        if (b < 0 || b >= B) { rc = -2; break; }\n", ""),
}

# Mutants of the bookkeeping model's slab-waste accounting (Python): each is
# the function's source with one mistake, run against the exact pins of
# test_oracle_bookkeeping.check_contiguous_reservation_waste.
WASTE_MUTANTS = {
    "live not clamped to the reservation": ("min(int(x), r)", "int(x)"),
    "live clamped the wrong way": ("min(int(x), r)", "max(int(x), r)"),
    "reserved counts one request too few": ("reserved = sum(reserve)", "reserved = sum(reserve[1:])"),
    "reserved off by one slot": ("reserved = sum(reserve)", "reserved = sum(reserve) + 1"),
    "wasted reversed": ('"wasted_slots": reserved - live', '"wasted_slots": live - reserved'),
    "one reservation for all, the first": ("reserve = [int(r) for r in reserve_tokens]",
                                           "reserve = [int(reserve_tokens[0])] * n"),
}


def _run_mutant(name, old, new, tmp):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique for {name!r}"
    tag = "".join(c if c.isalnum() else "_" for c in name)
    csrc = os.path.join(tmp, f"{tag}.c")
    lib = os.path.join(tmp, f"{tag}.so")
    with open(csrc, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", "-O1", "-std=c11", "-shared", "-fPIC", "-o", lib, csrc, "-lm"],
                   check=True, capture_output=True)
    env = dict(os.environ, PKV_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_mutant_is_caught():
    with tempfile.TemporaryDirectory() as tmp:
        with concurrent.futures.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 2)) as ex:
            results = list(ex.map(lambda kv: _run_mutant(kv[0], *kv[1], tmp), MUTANTS.items()))
    survivors = [name for name, rc in results if rc == 0]
    assert not survivors, f"pins did not catch: {survivors}"


def _waste_variant(old, new):
    import inspect
    import textwrap
    from oracle import bookkeeping
    src = textwrap.dedent(inspect.getsource(bookkeeping.contiguous_reservation_waste))
    assert src.count(old) == 1, old
    ns = {}
    exec(src.replace(old, new), ns)
    return ns["contiguous_reservation_waste"]


def test_every_waste_mutant_is_caught():
    from tests.test_oracle_bookkeeping import check_contiguous_reservation_waste
    check_contiguous_reservation_waste(_waste_variant("reserved = ", "reserved = "))
    survivors = []
    for name, (old, new) in WASTE_MUTANTS.items():
        try:
            check_contiguous_reservation_waste(_waste_variant(old, new))
        except AssertionError:
            continue
        survivors.append(name)
    assert not survivors, f"pins did not catch: {survivors}"


def test_unmutated_oracle_passes_under_the_same_harness():
    with tempfile.TemporaryDirectory() as tmp:
        name, rc = _run_mutant("identity", "#include <math.h>", "#include <math.h>", tmp)
    assert rc == 0
