"""Failure detection on the GPU without a fault: every pipeline wait in the
kernels is bounded.  A self-test launch waits on an mbarrier that nothing ever
arrives on, with each of the kernels' wait primitives; the wait must give up by
itself, report PKV_DEVERR_WAIT_TIMEOUT through the caller's flag, and leave the
context usable for the next call."""

import time

import pytest
import torch

import paged_kv_cache_360_b200 as pkv
from paged_kv_cache_360_b200 import _lib
from paged_kv_cache_360_b200.workloads import custom_workload
from tests.gpu_helpers import Dev, compare, ensure_built, oracle_decode

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    ensure_built()


@pytest.mark.parametrize("which", [0, 1, 2], ids=["decode-wait", "decode-abortable-wait", "prefill-wait"])
def test_bounded_wait_gives_up_and_the_context_stays_usable(which):
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    pkv.selftest_wait_timeout(which, err)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    print(f"wait {which} gave up after {elapsed:.3f} s")
    assert int(err.item()) == _lib.DEVERR_WAIT_TIMEOUT
    assert elapsed < 5.0
    # the next calls run normally on the same context
    wl = custom_workload(num_seqs=3, num_heads=8, num_kv_heads=2, head_dim=128, block_size=16,
                         context_lens=[1, 300, 1000], dtype=torch.bfloat16, seed=41)
    dev = Dev(wl)
    for P in (0, 128):
        out = dev.decode(P)
        assert int(dev.err.item()) == 0
        compare(out, oracle_decode(wl), what=f"decode after a timed-out wait, P={P}")
