"""Shared helpers of the GPU parity tests: move a workload to the device, run the
library's calls, run the oracle on the same host buffers, compare."""

import numpy as np
import torch

import oracle
import paged_kv_cache_360_b200 as pkv
from paged_kv_cache_360_b200 import _build

# Per element: |gpu - oracle| <= ATOL + RTOL * |oracle|  (oracle in float64).
ATOL = 2e-3
RTOL = 1e-2


def ensure_built():
    _build.build()


class Dev:
    """A workload's buffers on cuda:0."""

    def __init__(self, wl):
        self.wl = wl
        self.q = wl.q.cuda()
        self.k = wl.k_cache.cuda()
        self.v = wl.v_cache.cuda()
        self.tables = torch.from_numpy(np.ascontiguousarray(wl.block_tables)).cuda()
        self.lens = torch.from_numpy(np.ascontiguousarray(wl.context_lens)).cuda()
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")

    def decode(self, partition_size=0, tables=None, k=None, v=None):
        out = torch.empty_like(self.q)
        self.err.zero_()
        pkv.paged_attention_decode(out, self.q, self.k if k is None else k,
                                   self.v if v is None else v,
                                   self.tables if tables is None else tables, self.lens,
                                   self.wl.scale, partition_size=partition_size, err_flag=self.err)
        torch.cuda.synchronize()
        return out


def oracle_decode(wl, seqs=None, k=None, v=None, tables=None, threads=1):
    """The oracle's decode of the workload (float64 [B, H, D]).  With
    threads > 1 the sequences are shared out over that many threads, each
    calling the oracle on its own sequences (the C oracle runs outside the
    GIL); every output row is still the oracle's, computed the same way."""
    k = wl.k_cache if k is None else k
    v = wl.v_cache if v is None else v
    tables = wl.block_tables if tables is None else tables
    if threads <= 1:
        return oracle.paged_decode(wl.q, k, v, tables, wl.context_lens, wl.scale, seqs=seqs)
    import concurrent.futures
    todo = list(range(wl.num_seqs)) if seqs is None else [int(b) for b in seqs]
    shares = [[] for _ in range(threads)]
    loads = [0] * threads
    for b in sorted(todo, key=lambda b: -int(wl.context_lens[b])):
        i = loads.index(min(loads))
        shares[i].append(b)
        loads[i] += int(wl.context_lens[b]) + 1
    kw, vw = oracle.words(k), oracle.words(v)
    out = np.zeros((wl.num_seqs, wl.num_heads, wl.head_dim), dtype=np.float64)

    def run(share):
        part = oracle.paged_decode(wl.q, kw, vw, tables,
                                   wl.context_lens, wl.scale, seqs=sorted(share))
        return share, part

    with concurrent.futures.ThreadPoolExecutor(max_workers=threads) as ex:
        for share, part in ex.map(run, [s for s in shares if s]):
            out[share] = part[share]
    return out


PARITY_LOG = []


def report_parity(what, mabs, mrel, n, used):
    """Record and print one comparison's largest errors (the GPU tests' parity
    report): max abs, max rel (over |ref| > 1e-3) and the largest fraction of
    the per-element bound ATOL + RTOL |ref| used.  With PKV_PARITY_REPORT set,
    the run's records are also written there as JSON lines at the end of the
    session."""
    PARITY_LOG.append({"case": what, "max_abs": mabs, "max_rel": mrel, "tol_used": used,
                       "elements": n})
    print(f"parity {what}: max abs {mabs:.3e}, max rel {mrel:.3e}, {used:.2f} of the bound, "
          f"over {n} elements")


def compare(gpu_out, ref, seqs=None, what=""):
    g = gpu_out.detach().float().cpu().double().numpy()
    if seqs is not None:
        g, ref = g[seqs], ref[seqs]
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside {ATOL} + {RTOL}|ref|; "
            f"max abs {err.max():.3e}, first {idx.tolist()} gpu {g[bad][:5]} ref {ref[bad][:5]}")
    rel = err / np.maximum(np.abs(ref), 1e-30)
    mabs = float(err.max()) if err.size else 0.0
    mrel = float(np.where(np.abs(ref) > 1e-3, rel, 0).max()) if err.size else 0.0
    used = float((err / bound).max()) if err.size else 0.0
    if what:
        report_parity(what, mabs, mrel, int(err.size), used)
    return mabs, mrel


def words(t):
    return oracle.words(t)


def prefix_rows(tokens, Hkv, D, dtype):
    """K and V rows [len, Hkv, D] where the row at position p depends only on
    tokens[:p + 1] -- as a model's keys and values do, so that requests with the
    same prompt prefix have the same rows there."""
    from paged_kv_cache_360_b200.workloads import normal_tensor
    ks, vs = [], []
    for p in range(len(tokens)):
        rng = np.random.default_rng([7] + [int(t) for t in tokens[:p + 1]])
        ks.append(normal_tensor(rng, (Hkv, D), dtype))
        vs.append(normal_tensor(rng, (Hkv, D), dtype))
    return torch.stack(ks), torch.stack(vs)
