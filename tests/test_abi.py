"""The C-ABI library loads on a machine without a GPU and exports every function
include/pkv.h declares; host-side validation rejects bad arguments before any
CUDA work (no GPU needed for those paths)."""

import ctypes
import os
import re
import subprocess

import pytest

from paged_kv_cache_360_b200 import _build, _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return _lib.load()


def header_functions():
    text = open(os.path.join(ROOT, "include", "pkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                       text, flags=re.M)
    return sorted(set(n for n in names if n not in ("if", "return")))


def test_header_declares_what_the_binding_knows(lib):
    assert header_functions() == sorted(_lib.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, missing
    for n in header_functions():
        assert getattr(lib, n) is not None


def _desc(**kw):
    d = dict(num_blocks=8, block_size=16, num_kv_heads=2, head_dim=128, dtype=_lib.PKV_BF16)
    d.update(kw)
    return _lib.CacheDesc(d["num_blocks"], d["block_size"], d["num_kv_heads"], d["head_dim"], d["dtype"])


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: validation fails first


def _decode(lib, desc, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, mb=4, lens=FAKE, B=2, H=4, scale=0.1,
             P=0, ws=None, wsb=0)
    a.update(kw)
    return lib.paged_attention_decode(ctypes.byref(desc), a["out"], a["q"], a["k"], a["v"],
                                      a["tables"], a["mb"], a["lens"], a["B"], a["H"],
                                      ctypes.c_float(a["scale"]), a["P"], a["ws"], a["wsb"], None, None)


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), 2), (dict(block_size=8), 2), (dict(dtype=7), 2), (dict(num_blocks=0), 1),
    (dict(num_blocks=1 << 30, num_kv_heads=8), 2),
])
def test_decode_rejects_bad_descriptors(lib, kw, status):
    assert _decode(lib, _desc(**kw)) == status
    assert lib.pkv_last_error().decode()


def test_decode_rejects_bad_arguments(lib):
    d = _desc()
    assert _decode(lib, d, out=None) == 1
    assert _decode(lib, d, H=3) == 1                     # not a multiple of num_kv_heads
    assert _decode(lib, d, H=2 * 17) == 2                # group > 16
    assert _decode(lib, d, P=24) == 1                    # not a multiple of block_size
    assert _decode(lib, d, scale=float("nan")) == 1
    assert _decode(lib, d, q=ctypes.c_void_p(0x10002)) == 1   # misaligned
    assert _decode(lib, d, B=0) == 0                     # nothing to do
    # a split that needs a workspace, none given (without a device the balanced
    # part of the workspace cannot be sized: a CUDA error, nothing enqueued)
    assert _decode(lib, d, mb=64, P=128) == (5 if _has_device() else 4)


def _has_device():
    import torch
    return torch.cuda.is_available()


def test_workspace_size_formula(lib):
    d = _desc(head_dim=128, block_size=16)
    ws = lambda P: lib.paged_attention_workspace_bytes(ctypes.byref(d), 3, 4, 64, P)  # noqa: E731
    assert ws(1024) == 0 and ws(4096) == 0                 # fixed partitions, no split
    if not _has_device():
        assert ws(256) == 0 and ws(0) == 0                 # the balanced part needs the device
        return
    # the balanced workspace rounded up to 256 bytes, then the partition partials:
    # 64 blocks * 16 = 1024 tokens, P = 256 -> 4 partitions; (D + 2) floats per (b, h, p)
    balanced = ws(0)
    assert balanced > 0
    assert ws(256) == (balanced + 255) // 256 * 256 + 3 * 4 * 4 * 130 * 4


def test_append_and_copy_reject_bad_arguments(lib):
    d = _desc()
    assert lib.paged_kv_append(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, -1, None, None) == 1
    assert lib.paged_kv_append(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 0, None, None) == 0
    assert lib.paged_kv_append(ctypes.byref(d), FAKE, None, FAKE, FAKE, FAKE, 3, None, None) == 1
    assert lib.paged_kv_append(ctypes.byref(_desc(head_dim=80)), FAKE, FAKE, FAKE, FAKE, FAKE, 3,
                               None, None) == 2
    assert lib.copy_blocks(ctypes.byref(d), FAKE, FAKE, FAKE, -2, None, None) == 1
    assert lib.copy_blocks(ctypes.byref(d), FAKE, FAKE, FAKE, 0, None, None) == 0
    assert lib.copy_blocks(ctypes.byref(d), ctypes.c_void_p(0x10004), FAKE, FAKE, 2, None, None) == 1


def test_status_strings(lib):
    for code, name in _lib.STATUS_NAMES.items():
        assert lib.pkv_status_string(code).decode() == name


def test_selftest_rejects_bad_arguments(lib):
    # checked on the host before anything is launched
    assert lib.pkv_selftest_wait_timeout(3, FAKE, None) == 1
    assert lib.pkv_selftest_wait_timeout(-1, FAKE, None) == 1
    assert lib.pkv_selftest_wait_timeout(0, None, None) == 1
    assert "err_flag" in lib.pkv_last_error().decode()


def _prefill(lib, desc, **kw):
    a = dict(out=FAKE, q=FAKE, k=FAKE, v=FAKE, tables=FAKE, mb=4, lens=FAKE, qs=FAKE, B=2, T=40,
             H=4, scale=0.1)
    a.update(kw)
    return lib.paged_attention_prefill(ctypes.byref(desc), a["out"], a["q"], a["k"], a["v"],
                                       a["tables"], a["mb"], a["lens"], a["qs"], a["B"], a["T"],
                                       a["H"], ctypes.c_float(a["scale"]), None, None)


def test_prefill_rejects_bad_arguments(lib):
    d = _desc()
    assert _prefill(lib, _desc(head_dim=96)) == 2
    assert _prefill(lib, d, H=3) == 1                    # not a multiple of num_kv_heads
    assert _prefill(lib, d, H=6) == 2                    # group 3: not a power of two
    assert _prefill(lib, d, H=2 * 256) == 2              # group 256 > 128
    assert _prefill(lib, d, scale=float("inf")) == 1
    assert _prefill(lib, d, scale=-0.1) == 1
    assert _prefill(lib, d, T=-1) == 1
    assert _prefill(lib, d, mb=0) == 1
    assert _prefill(lib, d, qs=None) == 1
    assert _prefill(lib, d, out=ctypes.c_void_p(0x10008)) == 1   # misaligned
    assert _prefill(lib, d, out=ctypes.c_void_p(0x20000), q=ctypes.c_void_p(0x20400)) == 1  # overlap
    assert _prefill(lib, d, T=0) == 0                    # nothing to do
    assert _prefill(lib, d, B=0) == 0
    assert lib.pkv_last_error().decode()
