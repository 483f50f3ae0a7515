"""Benchmark of the paged decode step on B200: append + copy-on-write + decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl ours|reference]

One step = one pass of the whole hot path over one batch: the new token of every
sequence is appended through its slot (plus the block copies when the workload
shares blocks), then every sequence's query attends over its context through the
block table.  Inputs are resident in HBM before the timed region; the step is
captured once as a CUDA graph and replayed K times back to back, CUDA events on
the launching stream around the run (the value).  The decode kernels alone are
then replayed K times the same way (the roofline's average launch time).  The K/V read
per step (535 MB at the default workload) is 4x the 126 MB L2, so L2 is not
flushed between steps.

Multi-GPU (torchrun): each rank runs its own seeded batch (weak scaling, no
collective on the data path); times are the max over ranks.

``--impl reference`` times the CPU oracle on the host cores instead (bounded
samples of the same workload); under torchrun only rank 0 runs it.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s (% of B200 HBM peak); seq-decode-steps/sec"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


# ---------------------------------------------------------------- accounting

def decode_bytes(lens, wl) -> int:
    """Algorithmic bytes of one decode: K and V of every live token once, q, out,
    the block-table entries read and the lengths."""
    es = 2
    kv = int(np.sum(lens, dtype=np.int64)) * wl.num_kv_heads * wl.head_dim * es * 2
    qo = 2 * wl.num_seqs * wl.num_heads * wl.head_dim * es
    table = int(np.sum((np.asarray(lens, dtype=np.int64) + wl.block_size - 1) // wl.block_size)) * 4
    return kv + qo + table + 4 * wl.num_seqs


def unique_decode_bytes(lens, tables, wl) -> int:
    """decode_bytes with every physical K/V slot counted once: blocks shared by
    several sequences (a common prefix) are read from DRAM once, the rest of
    their reads hit L2."""
    bs = wl.block_size
    used = {}
    for b, L in enumerate(np.asarray(lens, dtype=np.int64)):
        for i in range(int((L + bs - 1) // bs)):
            blk = int(tables[b, i])
            used[blk] = max(used.get(blk, 0), int(min(bs, L - i * bs)))
    kv = sum(used.values()) * wl.num_kv_heads * wl.head_dim * 2 * 2
    return decode_bytes(lens, wl) - int(np.sum(lens, dtype=np.int64)) * wl.num_kv_heads * wl.head_dim * 4 + kv


def append_bytes(n_tokens, wl) -> int:
    row = wl.num_kv_heads * wl.head_dim * 2
    return n_tokens * (2 * row * 2 + 8)        # read key+value, write them, read the slot


def copy_bytes(n_pairs, wl) -> int:
    block = wl.num_kv_heads * wl.block_size * wl.head_dim * 2
    return n_pairs * (2 * 2 * block + 8)       # K and V: read + write, read the pair


# --------------------------------------------------------------- multi-rank

def max_over_ranks(values, world, device=None):
    """Max of each value over all ranks (device times: the slowest rank decides)."""
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def whole_job_gbs(bytes_per_rank_step, world, ms_per_step) -> float:
    """Aggregate throughput: every rank processes its own batch in the same step time."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------ workload

def _reserve_step(pool, seqs, counts):
    """One step's reservations: the block manager's batched call when it has
    one, else one reserve per sequence in order (the two agree bit for bit)."""
    if hasattr(pool, "reserve_batch"):
        sl, cp = pool.reserve_batch(seqs, counts)
        return [int(x) for x in sl], [tuple(p) for p in cp]
    slots, pairs = [], []
    for i, s in enumerate(seqs):
        sl, cp = pool.reserve(s, 1 if counts is None else int(counts[i]))
        slots.extend(int(x) for x in sl)
        pairs.extend(tuple(p) for p in cp)
    return slots, pairs


def _tables(pool, seqs):
    mb = max(len(pool.table(s)) for s in seqs)
    tables = np.full((len(seqs), mb), -1, dtype=np.int32)
    for i, s in enumerate(seqs):
        t = pool.table(s)
        tables[i, :len(t)] = t
    lens = np.array([pool.length(s) for s in seqs], dtype=np.int32)
    return tables, lens


def build_step(wl, make_pool):
    """Host bookkeeping for one decode step.

    ``make_pool(num_blocks, block_size, free_order)`` gives the block manager:
    the library's ``Pool`` on our arm, the oracle's ``BlockPoolModel`` on the
    reference arm (the two agree bit for bit, tests/test_pool_parity.py).
    Returns (pairs, slots, tables, lens, key, value): the copy pairs, the slots
    of the appended tokens, the block tables and lengths the decode reads, and
    the keys/values appended."""
    bs = wl.block_size
    pool = make_pool(wl.num_blocks, bs, wl.free_order)
    pairs, slots = [], []
    if wl.prefix_len:
        s0 = pool.new_seq()
        pool.reserve(s0, wl.prefix_len)
        seqs = [s0] + [pool.fork(s0) for _ in range(wl.num_seqs - 1)]
        last_prefix_block = (wl.prefix_len + bs - 1) // bs - 1
        for s in seqs:
            p = pool.cow(s, last_prefix_block)
            if p:
                pairs.append(tuple(p))
        sl, cp = _reserve_step(pool, seqs, [int(n) + 1 for n in wl.suffix_lens[:len(seqs)]])
    else:
        seqs = []
        for b in range(wl.num_seqs):
            s = pool.new_seq()
            pool.reserve(s, int(wl.context_lens[b]) - 1)
            seqs.append(s)
        # the step's allocation, one call for the whole batch
        sl, cp = _reserve_step(pool, seqs, None)
    pairs.extend(cp)
    slots.extend(sl)
    tables, lens = _tables(pool, seqs)
    if hasattr(pool, "close"):
        pool.close()
    return (np.array(pairs, dtype=np.int32).reshape(-1, 2), np.array(slots, dtype=np.int64),
            tables, lens, wl.new_key, wl.new_value)


def library_pool(pkv):
    return lambda nb, bs, order: pkv.Pool(nb, bs, order)


def oracle_pool():
    import oracle
    return lambda nb, bs, order: oracle.BlockPoolModel(nb, bs, order)


# ------------------------------------------------------------------- clocks

class ClockSampler:
    def __init__(self, period_ms=20):
        self.period_ms = period_ms
        self.rows = []
        self.proc = None
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_FIELDS}", "--format=csv,noheader,nounits",
                 f"-lms={self.period_ms}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark(self, name):
        self.marks.append((name, time.time()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1):
        inside = [r for t, r in self.rows if t0 <= t <= t1]
        window = "timed region"
        if len(inside) < 3:
            inside = [r for t, r in self.rows]
            window = "whole run (timed region shorter than the sampling period)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in inside if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in inside if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i in range(4)
                          if len(r) > 5 + i and r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(inside), "window": window}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def decode_device_sha256() -> str:
    """Hash of the decode kernels' device code: pkv_decode.cu up to its host
    section, and the device headers it includes."""
    import hashlib
    csrc = os.path.join(ROOT, "paged_kv_cache_360_b200", "csrc")
    h = hashlib.sha256()
    src = open(os.path.join(csrc, "pkv_decode.cu"), "rb").read()
    h.update(src[:src.find(b"// ------------------------------------------------------------------ host side")])
    for name in ("pkv_attend.cuh", "pkv_ptx.cuh", "pkv_cascade.cuh"):
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()


def prefill_device_sha256() -> str:
    """Hash of the prefill kernel's device code: pkv_prefill.cu up to its host
    section, and the device headers it includes."""
    import hashlib
    csrc = os.path.join(ROOT, "paged_kv_cache_360_b200", "csrc")
    h = hashlib.sha256()
    src = open(os.path.join(csrc, "pkv_prefill.cu"), "rb").read()
    h.update(src[:src.find(b"// ------------------------------------------------------------------ host side")])
    for name in ("pkv_tc.cuh", "pkv_ptx.cuh", "pkv_wait.cuh"):
        h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()


def read_record(name, sha):
    """bytes_per_launch from a committed ncu summary profiles/<name> taken on
    device code with the given hash (else None)."""
    try:
        rec = {}
        for line in open(os.path.join(ROOT, "profiles", name)):
            if ":" in line and not line.startswith("#"):
                key, val = line.split(":", 1)
                rec[key.strip()] = val.strip()
    except OSError:
        return None
    if rec.get("source_sha256") != sha:
        return None
    return int(rec["bytes_per_launch"])


def traffic_record():
    """DRAM bytes per decode launch from the committed ncu summary
    profiles/decode_traffic.txt, if it was taken on the current decode source
    (else None)."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.txt")
    try:
        rec = {}
        for line in open(path):
            if ":" in line and not line.startswith("#"):
                key, val = line.split(":", 1)
                rec[key.strip()] = val.strip()
    except OSError:
        return None
    if rec.get("source_sha256") != decode_device_sha256():
        return None
    return {"bytes_per_launch": int(rec["bytes_per_launch"])}


# ---------------------------------------------------------------- our arm

def run_ours(args, rank, world, local_rank):
    import paged_kv_cache_360_b200 as pkv
    from paged_kv_cache_360_b200.workloads import make_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = make_workload(args.config, seed=args.seed, rank=rank)
    pairs, slots, tables, lens, new_key, new_value = build_step(wl, library_pool(pkv))

    k = wl.k_cache.to(dev)
    v = wl.v_cache.to(dev)
    q = wl.q.to(dev)
    d_key, d_value = new_key.to(dev), new_value.to(dev)
    d_slots = torch.from_numpy(slots).to(dev)
    d_pairs = torch.from_numpy(pairs).to(dev)
    d_tables = torch.from_numpy(tables).to(dev)
    d_lens = torch.from_numpy(lens).to(dev)
    out = torch.empty_like(q)
    B, H = wl.num_seqs, wl.num_heads
    P = args.partition_size if args.partition_size is not None else wl.partition_size
    shared = args.shared_prefix and wl.prefix_len > 0
    if shared:
        # groups of sequences that share their tables' leading blocks
        group_start, group_blocks = pkv.shared_prefix_groups(tables, lens, wl.block_size)
        ws_bytes = pkv.paged_attention_shared_prefix_workspace_bytes(k, B, H, tables.shape[1],
                                                                      group_start, group_blocks)
    else:
        ws_bytes = pkv.paged_attention_workspace_bytes(k, B, H, tables.shape[1], P)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def decode_call(o, q_, t_, l_):
        if shared:
            pkv.paged_attention_decode_shared_prefix(o, q_, k, v, t_, l_, wl.scale, group_start,
                                                     group_blocks, workspace=ws, err_flag=err)
        else:
            pkv.paged_attention_decode(o, q_, k, v, t_, l_, wl.scale, partition_size=P,
                                       workspace=ws, err_flag=err)

    def step_write():
        if len(pairs):
            pkv.copy_blocks(k, v, d_pairs, err_flag=err)
        pkv.paged_kv_append(k, v, d_key, d_value, d_slots, err_flag=err)

    def step_decode():
        decode_call(out, q, d_tables, d_lens)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        n0 = pkv.launch_count()
        step_write()
        step_decode()
        launches_per_step = pkv.launch_count() - n0
    torch.cuda.synchronize()
    # the whole step as one graph (append [+ copies] and decode, the decode
    # launched as a programmatic dependent of the append), and the decode alone
    g_step, g_decode = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        step_write()
        step_decode()
    with torch.cuda.graph(g_decode, stream=stream):
        step_decode()
    torch.cuda.synchronize()

    step_bytes_decode = decode_bytes(lens, wl)
    step_bytes = step_bytes_decode + append_bytes(len(slots), wl) + copy_bytes(len(pairs), wl)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    spread = {}

    def timed(graph, steps, name=None):
        """Device time (ms) of `steps` back-to-back replays: CUDA events on the
        launching stream around the whole run, barrier + synchronize on both
        sides.  Events also split the run into up to 20 equal chunks, whose
        per-step times give the p10 / median / p90 spread (under `name`)."""
        chunks = max(1, min(20, steps))
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(chunks + 1)]
        bounds = [steps * c // chunks for c in range(chunks + 1)]
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            marks[0].record(stream)
            for c in range(chunks):
                for _ in range(bounds[c + 1] - bounds[c]):
                    graph.replay()
                marks[c + 1].record(stream)
        torch.cuda.synchronize()
        barrier()
        if name:
            per = sorted(marks[c].elapsed_time(marks[c + 1]) / (bounds[c + 1] - bounds[c])
                         for c in range(chunks) if bounds[c + 1] > bounds[c])
            spread[name] = {"p10": round(per[len(per) // 10], 5), "median": round(per[len(per) // 2], 5),
                            "p90": round(per[(len(per) * 9) // 10 - (1 if len(per) >= 10 else 0)], 5),
                            "chunks": len(per)}
        return marks[0].elapsed_time(marks[-1])

    sampler = ClockSampler()
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_step.replay()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    step_ms = timed(g_step, args.steps, "step_ms")      # the timed region: K whole steps
    t_wall1 = time.time()
    decode_ms = timed(g_decode, args.steps, "decode_ms")  # the dominant kernels alone, K launches

    # End to end through the public API: every step copies its inputs from
    # pinned host memory to the device, runs the library's calls and reads the
    # output back to pinned host memory, all on one stream.  Measured twice:
    # the step captured as one CUDA graph (the copies are graph nodes, as a
    # serving engine would run it), and plain eager calls.
    # The step's inputs are staged in one page-locked buffer and copied with one
    # host -> device copy into one device buffer the library's calls read through
    # views (each input 256-byte aligned).
    inputs = [("q", wl.q), ("key", new_key), ("value", new_value), ("slots", torch.from_numpy(slots)),
              ("tables", torch.from_numpy(tables)), ("lens", torch.from_numpy(lens))]
    if len(pairs):
        inputs.append(("pairs", torch.from_numpy(pairs)))
    offsets, total = {}, 0
    for name, t in inputs:
        offsets[name] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    h_stage = torch.empty(total, dtype=torch.uint8).pin_memory()
    d_stage = torch.empty(total, dtype=torch.uint8, device=dev)

    def view(buf, name, t):
        nbytes = t.numel() * t.element_size()
        return buf[offsets[name]:offsets[name] + nbytes].view(t.dtype).view(t.shape)

    for name, t in inputs:
        view(h_stage, name, t).copy_(t)
    dv = {name: view(d_stage, name, t) for name, t in inputs}
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_out = torch.empty_like(out)
    h2d = total
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step():
        d_stage.copy_(h_stage, non_blocking=True)
        if len(pairs):
            pkv.copy_blocks(k, v, dv["pairs"], err_flag=err)
        pkv.paged_kv_append(k, v, dv["key"], dv["value"], dv["slots"], err_flag=err)
        decode_call(e2e_out, dv["q"], dv["tables"], dv["lens"])
        h_out.copy_(e2e_out, non_blocking=True)

    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=stream):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 2000))
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_e2e.replay()
    e2e_serial_ms = timed(g_e2e, e2e_steps)

    # The same steps pipelined, as a serving loop runs them: inputs and outputs
    # double-buffered, step i+1's host -> device copy on one copy stream and
    # step i's device -> host copy on another while step i's kernels run.
    # PIPE steps (their cross-stream dependencies as event edges) are one CUDA
    # graph; every step still copies its inputs in and its output out.
    PIPE = 16
    h_stages = [h_stage, torch.empty_like(h_stage).pin_memory()]
    h_stages[1].copy_(h_stage)
    d_stages = [d_stage, torch.empty_like(d_stage)]
    dvs = [{name: view(d_stages[j], name, t) for name, t in inputs} for j in range(2)]
    outs = [e2e_out, torch.empty_like(out)]
    h_outs = [h_out, torch.empty_like(h_out).pin_memory()]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def pipelined_steps():
        fork = torch.cuda.Event()
        fork.record(stream)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        ev_comp, ev_read = [], []
        for i in range(PIPE):
            j = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])      # step i-2 is done with d_stages[j]
                d_stages[j].copy_(h_stages[j], non_blocking=True)
                ev_in = torch.cuda.Event()
                ev_in.record(s_in)
            stream.wait_event(ev_in)
            if i >= 2:
                stream.wait_event(ev_read[i - 2])        # outs[j] of step i-2 has been read
            d = dvs[j]
            if len(pairs):
                pkv.copy_blocks(k, v, d["pairs"], err_flag=err)
            pkv.paged_kv_append(k, v, d["key"], d["value"], d["slots"], err_flag=err)
            decode_call(outs[j], d["q"], d["tables"], d["lens"])
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            ev_comp.append(ev_c)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_c)
                h_outs[j].copy_(outs[j], non_blocking=True)
                ev_r = torch.cuda.Event()
                ev_r.record(s_out)
                ev_read.append(ev_r)
        stream.wait_event(ev_in)
        stream.wait_event(ev_read[-1])

    g_pipe = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_pipe, stream=stream):
        pipelined_steps()
    torch.cuda.synchronize()
    pipe_replays = max(1, e2e_steps // PIPE)
    with torch.cuda.stream(stream):
        for _ in range(max(1, args.warmup // PIPE)):
            g_pipe.replay()
    e2e_ms = timed(g_pipe, pipe_replays)
    e2e_pipe_steps = pipe_replays * PIPE
    eager_steps = max(3, min(args.steps, 200))
    eager_ms = 0.0
    barrier()
    with torch.cuda.stream(stream):
        for i in range(args.warmup + eager_steps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            e2e_step()
            e1.record(stream)
            e1.synchronize()          # the host reads the step's output
            if i >= args.warmup:
                eager_ms += e0.elapsed_time(e1)
    barrier()
    if rank == 0:
        sampler.stop()
    torch.cuda.synchronize()
    err_val = int(err.item())

    step_ms, decode_ms, e2e_ms, e2e_serial_ms, eager_ms = max_over_ranks(
        [step_ms, decode_ms, e2e_ms, e2e_serial_ms, eager_ms], world, dev)
    if rank != 0:
        return None

    peak, peak_kind = measured_peak()
    ms_per_step = step_ms / args.steps
    value = whole_job_gbs(step_bytes, world, ms_per_step)
    decode_avg_ms = decode_ms / args.steps
    achieved = step_bytes_decode / (decode_avg_ms * 1e-3) / 1e9
    # the committed record is one balanced-decode launch of the llama3-8b-layer workload
    traffic = traffic_record() if (wl.config == 2 and P == 0 and not shared) else None
    e2e_per_step = e2e_ms / e2e_pipe_steps
    serial_per_step = e2e_serial_ms / e2e_steps
    eager_per_step = eager_ms / eager_steps
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f16",
        "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs_per_gpu": B, "global_num_seqs": B * world,
                   "num_heads": H, "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                   "block_size": wl.block_size, "num_blocks": wl.num_blocks,
                   "mean_context_len": float(np.mean(lens)), "max_context_len": int(np.max(lens)),
                   "partition_size": int(P),
                   "schedule": ("shared-prefix decode, groups %s sharing %s blocks"
                                % ([int(x) for x in group_start], [int(x) for x in group_blocks]))
                               if shared else
                               "balanced" if P == 0 else f"fixed partitions of {P} tokens",
                   "copy_pairs": int(len(pairs)),
                   "appended_tokens": int(len(slots)), "seed": args.seed,
                   "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": "not flushed: the step reads %.0f MB of K/V, %.1fx the 126 MB L2"
                         % (step_bytes_decode / 1e6, step_bytes_decode / 126e6),
                   "timing": "CUDA events around K back-to-back replays of the step's CUDA graph"},
        "seq_decode_steps_per_s": round(world * B / (ms_per_step * 1e-3), 1),
        "hbm_frac": round(value / world / peak, 4),
        "hbm_frac_of_nominal_7700": round(value / world / 7700.0, 4),
        "decode_unique_bytes_gbs": round(unique_decode_bytes(lens, tables, wl) / (decode_avg_ms * 1e-3) / 1e9, 2),
        "spread_ms_per_step": spread,
        "algorithmic_bytes_per_step": step_bytes,
        "roofline": {"bound": "hbm",
                     "kernel": "paged_attention_decode_shared_prefix (balanced decode of the own "
                               "tokens, chain merge, tcgen05 prefix tiles, final merge)" if shared else
                               "paged_attention_decode (balanced decode + chain-merge kernels)"
                               if P == 0 else "paged_attention_decode (partition + reduce kernels)",
                     "timing": "CUDA events around K back-to-back decode-only graph replays",
                     "achieved": round(achieved, 2), "peak": peak, "peak_kind": peak_kind,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": None if traffic is None else traffic["bytes_per_launch"],
                     "algorithmic_bytes_per_launch": step_bytes_decode,
                     "avg_launch_ms": round(decode_avg_ms, 5)},
        "e2e": {"value": round(whole_job_gbs(step_bytes, world, e2e_per_step), 2), "unit": "GB/s",
                "ms_per_step": round(e2e_per_step, 5), "steps": e2e_pipe_steps,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "per step: one pinned host -> device copy of the step's inputs (q, new K/V, "
                        "slots, tables, lengths, staged in one buffer); paged_kv_append; "
                        "paged_attention_decode; device -> pinned host copy of the output.  Inputs "
                        "and outputs double-buffered: the copies run on two copy streams beside "
                        "the kernels of the neighbouring steps; %d steps per CUDA graph" % PIPE,
                "serial": {"value": round(whole_job_gbs(step_bytes, world, serial_per_step), 2),
                           "ms_per_step": round(serial_per_step, 5), "steps": e2e_steps,
                           "path": "the same step with its copies and kernels on one stream, one "
                                   "step per CUDA graph"},
                "eager": {"value": round(whole_job_gbs(step_bytes, world, eager_per_step), 2),
                          "ms_per_step": round(eager_per_step, 5), "steps": eager_steps,
                          "path": "the same calls issued eagerly from Python, host waits for "
                                  "the output every step"}},
        "gpu_launches": int(launches_per_step * args.steps),
        "launches_per_step": int(launches_per_step),
        "device_err_flag": err_val,
        "clocks": sampler.summary(t_wall0, t_wall1),
    }
    if world == 1 and not args.no_extras:
        line.update(extra_records(pkv, dev, peak, args.seed))
    if world == 1 and not args.no_cpu_baseline:
        one = cpu_baseline(wl, lens, tables, slots, new_key, new_value, budget_s=args.cpu_budget)
        try:
            allc = cpu_baseline_all_cores(wl, lens, one["sample_seqs"])
            line["cpu_baseline"] = dict(one, value=allc["value"], cores=allc["cores"],
                                        seconds=allc["seconds"],
                                        single_core={"value": one["value"], "seconds": one["seconds"]},
                                        sample=one["sample"] + f"; timed on {allc['cores']} spawned "
                                               "processes, one share each, value = sample bytes / "
                                               "slowest process")
        except Exception as e:  # the single-core figure stands on its own
            line["cpu_baseline"] = dict(one, all_cores_error=str(e)[:200])
    return line


# ------------------------------------------------------------ extra records

def _device_values(shape, dtype, dev, gen):
    """N(0, 1) values drawn on the device.  The extra records below time
    kernels whose run time does not depend on the values, so their K/V/q are
    drawn here instead of by the host generator (which takes minutes for a
    1 GB pool); shapes, lengths and block tables are the workload's own."""
    return torch.randn(shape, generator=gen, device=dev, dtype=torch.float32).to(dtype)


class _Timer:
    """Device time of one captured call: CUDA events on its stream."""

    def __init__(self, dev, stream):
        self.dev, self.stream = dev, stream
        self.flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)   # 2x the 126 MB L2

    def capture(self, fn):
        with torch.cuda.stream(self.stream):
            fn()                       # eager once (first-call set-up)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            fn()
        torch.cuda.synchronize()
        return g

    def back_to_back(self, fn, steps, warmup=5):
        """Average ms of `steps` replays back to back (inputs larger than L2)."""
        g = self.capture(fn)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                g.replay()
            e0.record(self.stream)
            for _ in range(steps):
                g.replay()
            e1.record(self.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / steps

    def flushed(self, fn, steps, warmup=3):
        """Average ms of one call with L2 flushed before each (a 256 MB write
        between calls, outside the events): for inputs that fit in L2."""
        g = self.capture(fn)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                self.flush.zero_()
                g.replay()
            for e0, e1 in ev:
                self.flush.zero_()
                e0.record(self.stream)
                g.replay()
                e1.record(self.stream)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / steps


def extra_records(pkv, dev, peak, seed):
    """Kernels of the path beyond the headline workload, each in its own short
    timed region: the decode on the shared-prefix, long-context and
    70B-shaped workloads (both schedules where the workload names one), the
    paged prefill, and the data-movement kernels (append, copy_blocks,
    swap_blocks)."""
    from paged_kv_cache_360_b200.workloads import make_workload, make_prefill_workload
    stream = torch.cuda.Stream(device=dev)
    timer = _Timer(dev, stream)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + int(seed))
    out = {}

    # ---- decode on the other workloads
    by_wl = {}
    for config, P in ((3, 0), (4, 512), (4, 0), (5, 0), (5, 512)):
        wl = make_workload(config, seed=seed, materialize=False)
        if config == 3:
            _, _, tables, lens, _, _ = build_step(wl, library_pool(pkv))
        else:
            tables, lens = wl.block_tables, wl.context_lens
        B, H, D = wl.num_seqs, wl.num_heads, wl.head_dim
        shape = (wl.num_blocks, wl.num_kv_heads, wl.block_size, D)
        k = _device_values(shape, wl.dtype, dev, gen)
        v = _device_values(shape, wl.dtype, dev, gen)
        q = _device_values((B, H, D), wl.dtype, dev, gen)
        o = torch.empty_like(q)
        d_t = torch.from_numpy(np.ascontiguousarray(tables)).to(dev)
        d_l = torch.from_numpy(np.ascontiguousarray(lens)).to(dev)
        ws = torch.empty(max(16, pkv.paged_attention_workspace_bytes(k, B, H, d_t.shape[1], P)),
                         dtype=torch.uint8, device=dev)
        err = torch.zeros(1, dtype=torch.int32, device=dev)

        def decode():
            pkv.paged_attention_decode(o, q, k, v, d_t, d_l, wl.scale, partition_size=P,
                                       workspace=ws, err_flag=err)

        nbytes = decode_bytes(lens, wl)
        fits_l2 = unique_decode_bytes(lens, tables, wl) < 126e6
        ms = timer.flushed(decode, 100) if fits_l2 else timer.back_to_back(decode, 200)
        if config == 3:
            # the same batch through the shared-prefix decode: the groups come
            # from the tables (every sequence shares the prompt's full blocks)
            gs, gb = pkv.shared_prefix_groups(tables, lens, wl.block_size)
            ws_sp = torch.empty(max(256, pkv.paged_attention_shared_prefix_workspace_bytes(
                k, B, H, d_t.shape[1], gs, gb)), dtype=torch.uint8, device=dev)
            o_sp = torch.empty_like(q)

            def decode_sp():
                pkv.paged_attention_decode_shared_prefix(o_sp, q, k, v, d_t, d_l, wl.scale, gs, gb,
                                                         workspace=ws_sp, err_flag=err)

            ms_sp = timer.flushed(decode_sp, 100)
            ub = unique_decode_bytes(lens, tables, wl)
            by_wl["3_shared_prefix"] = {
                "workload": wl.name, "schedule": "shared-prefix decode (prefix tiles on tcgen05 + "
                                                 "balanced decode of each sequence's own tokens)",
                "groups": {"group_start": [int(x) for x in gs], "shared_blocks": [int(x) for x in gb]},
                "num_seqs": B, "ms": round(ms_sp, 5), "algorithmic_bytes": nbytes,
                "gbs": round(nbytes / (ms_sp * 1e-3) / 1e9, 1),
                "frac": round(nbytes / (ms_sp * 1e-3) / 1e9 / peak, 4),
                "unique_bytes": ub, "unique_gbs": round(ub / (ms_sp * 1e-3) / 1e9, 1),
                "unique_frac": round(ub / (ms_sp * 1e-3) / 1e9 / peak, 4),
                "speedup_vs_balanced": round(ms / ms_sp, 3),
                "seq_decode_steps_per_s": round(B / (ms_sp * 1e-3), 1),
                "timing": "L2 flushed before each launch, events around it"}
        rec = {"workload": wl.name, "schedule": "balanced" if P == 0 else f"fixed partitions of {P}",
               "num_seqs": B, "ms": round(ms, 5), "algorithmic_bytes": nbytes,
               "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
               "frac": round(nbytes / (ms * 1e-3) / 1e9 / peak, 4),
               "seq_decode_steps_per_s": round(B / (ms * 1e-3), 1),
               "timing": "L2 flushed before each launch, events around it" if fits_l2
                         else "events around 200 back-to-back decode-only replays",
               "device_err_flag": int(err.item())}
        if config == 3:
            ub = unique_decode_bytes(lens, tables, wl)
            rec["unique_bytes"] = ub
            rec["unique_gbs"] = round(ub / (ms * 1e-3) / 1e9, 1)
            rec["bytes_note"] = ("algorithmic bytes count the shared prefix once per sequence; "
                                 "unique bytes count every physical slot once")
        by_wl[f"{config}" if P == wl.partition_size else f"{config}_{'balanced' if P == 0 else f'fixed{P}'}"] = rec
        del k, v, q, o, ws
        torch.cuda.empty_cache()
    out["decode_by_workload"] = by_wl

    # ---- paged prefill
    pw = make_prefill_workload("prefill-llama3-8b-layer", seed=seed, materialize=False)
    slots, tables, lens = build_prefill_step(pw, library_pool(pkv))
    T, H, D = pw.num_tokens, pw.num_heads, pw.head_dim
    shape = (pw.num_blocks, pw.num_kv_heads, pw.block_size, D)
    k = _device_values(shape, pw.dtype, dev, gen)
    v = _device_values(shape, pw.dtype, dev, gen)
    q = _device_values((T, H, D), pw.dtype, dev, gen)
    o = torch.empty_like(q)
    d_t = torch.from_numpy(tables).to(dev)
    d_l = torch.from_numpy(lens).to(dev)
    d_qs = torch.from_numpy(pw.query_start).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def prefill():
        pkv.paged_attention_prefill(o, q, k, v, d_t, d_l, d_qs, pw.scale, err_flag=err)

    ms = timer.back_to_back(prefill, 50)
    flops = prefill_flops(lens, pw.query_start, H, D)
    tpeak, tpeak_sustained, tkind = measured_tensor_peak()
    tf = flops / (ms * 1e-3) / 1e12
    out["prefill"] = {"workload": pw.name, "unit": "TFLOP/s", "value": round(tf, 2),
                      "avg_launch_ms": round(ms, 5), "algorithmic_flops_per_launch": flops,
                      "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": tpeak,
                                   "peak_kind": f"{tkind} bf16 dense burst", "frac": round(tf / tpeak, 4),
                                   "peak_sustained": tpeak_sustained,
                                   "frac_of_sustained": round(tf / tpeak_sustained, 4)
                                   if tpeak_sustained else None},
                      "timing": "events around 50 back-to-back prefill-only replays "
                                "(the pool is 179 MB, larger than L2)",
                      "device_err_flag": int(err.item())}
    del k, v, q, o
    torch.cuda.empty_cache()

    # ---- data movement: the shared-prefix step's append and copies, a swap
    wl = make_workload(3, seed=seed, materialize=False)
    pairs, slots, _, _, _, _ = build_step(wl, library_pool(pkv))
    shape = (wl.num_blocks, wl.num_kv_heads, wl.block_size, wl.head_dim)
    k = _device_values(shape, wl.dtype, dev, gen)
    v = _device_values(shape, wl.dtype, dev, gen)
    n_new = len(slots)
    key = _device_values((n_new, wl.num_kv_heads, wl.head_dim), wl.dtype, dev, gen)
    val = _device_values((n_new, wl.num_kv_heads, wl.head_dim), wl.dtype, dev, gen)
    d_slots = torch.from_numpy(slots).to(dev)
    d_pairs = torch.from_numpy(pairs).to(dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    moves = {}
    ms = timer.flushed(lambda: pkv.paged_kv_append(k, v, key, val, d_slots, err_flag=err), 100)
    nb = append_bytes(n_new, wl)
    moves["append"] = {"what": f"paged_kv_append of the {wl.name} step ({n_new} tokens)",
                       "ms": round(ms, 5), "bytes": nb, "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                       "frac_hbm": round(nb / (ms * 1e-3) / 1e9 / peak, 4)}
    ms = timer.flushed(lambda: pkv.copy_blocks(k, v, d_pairs, err_flag=err), 100)
    nb = copy_bytes(len(pairs), wl)
    moves["copy_blocks"] = {"what": f"copy_blocks of the {wl.name} step ({len(pairs)} pairs)",
                            "ms": round(ms, 5), "bytes": nb, "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                            "frac_hbm": round(nb / (ms * 1e-3) / 1e9 / peak, 4)}
    # a larger pool of the same geometry (4096 blocks, 128 MiB per K or V pool)
    # for a 1024-pair copy and a 1024-block swap
    del k, v
    rng = np.random.default_rng(seed)
    shape = (4096,) + shape[1:]
    k = _device_values(shape, wl.dtype, dev, gen)
    v = _device_values(shape, wl.dtype, dev, gen)
    # distinct destinations that are never sources (the pairs a block manager emits)
    ids = rng.permutation(shape[0])
    big = np.stack([ids[:1024], ids[1024:2048]], 1).astype(np.int32)
    d_big = torch.from_numpy(big).to(dev)
    ms = timer.flushed(lambda: pkv.copy_blocks(k, v, d_big, err_flag=err), 50)
    nb = copy_bytes(len(big), wl)
    moves["copy_blocks_1024"] = {"what": "copy_blocks of 1024 random pairs (64 MiB read, 64 MiB "
                                         "written) in a 4096-block pool of the same geometry",
                                 "ms": round(ms, 5), "bytes": nb, "gbs": round(nb / (ms * 1e-3) / 1e9, 1),
                                 "frac_hbm": round(nb / (ms * 1e-3) / 1e9 / peak, 4)}
    n_swap = 1024
    blk_bytes = wl.num_kv_heads * wl.block_size * wl.head_dim * 2
    lst = torch.from_numpy(ids[:n_swap].astype(np.int32)).to(dev)
    hk = torch.empty((n_swap,) + shape[1:], dtype=wl.dtype).pin_memory()
    hv = torch.empty((n_swap,) + shape[1:], dtype=wl.dtype).pin_memory()
    link_bytes = 2 * n_swap * blk_bytes
    dbuf = torch.empty(link_bytes, dtype=torch.uint8, device=dev)
    hbuf = torch.empty(link_bytes, dtype=torch.uint8).pin_memory()
    ms_d2h = timer.flushed(lambda: hbuf.copy_(dbuf, non_blocking=True), 20)
    ms_h2d = timer.flushed(lambda: dbuf.copy_(hbuf, non_blocking=True), 20)
    for name, to_host, ref_ms in (("swap_out", True, ms_d2h), ("swap_in", False, ms_h2d)):
        ms = timer.flushed(lambda: pkv.swap_blocks(k, v, hk, hv, lst, to_host, err_flag=err), 20)
        link = link_bytes / (ref_ms * 1e-3) / 1e9
        moves[name] = {"what": f"swap_blocks of {n_swap} blocks "
                               f"({'device -> pinned host' if to_host else 'pinned host -> device'}, "
                               f"{link_bytes >> 20} MiB)",
                       "ms": round(ms, 5), "bytes_over_link": link_bytes,
                       "gbs": round(link_bytes / (ms * 1e-3) / 1e9, 2),
                       "link_copy_gbs": round(link, 2),
                       "frac_of_link_copy": round(link_bytes / (ms * 1e-3) / 1e9 / link, 4),
                       "link_copy": "one cudaMemcpyAsync of the same bytes, contiguous, pinned"}
    moves["device_err_flag"] = int(err.item())
    moves["timing"] = "L2 flushed before each launch, events around it"
    out["data_movement"] = moves
    return out


# ------------------------------------------------------------------ prefill

PREFILL_METRIC = "paged prefill attention TFLOP/s (causal, % of B200 bf16 dense peak)"


def build_prefill_step(wl, make_pool):
    """Block tables, lengths and the query tokens' slots from a block manager
    (``make_pool`` as in build_step): every sequence first holds its earlier
    context, then reserves its query tokens."""
    pool = make_pool(wl.num_blocks, wl.block_size, wl.free_order)
    seqs = []
    nq = np.diff(wl.query_start)
    for b in range(wl.num_seqs):
        s = pool.new_seq()
        pool.reserve(s, int(wl.context_lens[b] - nq[b]))
        seqs.append(s)
    slots = []
    for b, s in enumerate(seqs):
        sl, cp = pool.reserve(s, int(nq[b]))
        assert not cp
        slots.extend(int(x) for x in sl)
    tables, lens = _tables(pool, seqs)
    if hasattr(pool, "close"):
        pool.close()
    return np.asarray(slots, dtype=np.int64), tables, lens


def prefill_flops(lens, query_start, H, D) -> int:
    """Causal attention FLOPs: 2 D for q . k and 2 D for p v per (query row,
    visible key) pair and head."""
    nq = np.diff(np.asarray(query_start, dtype=np.int64))
    L = np.asarray(lens, dtype=np.int64)
    pairs = nq * (L - nq) + nq * (nq + 1) // 2
    return int(pairs.sum()) * 4 * H * D


def measured_tensor_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0.0)), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def run_prefill(args, rank, world, local_rank):
    import paged_kv_cache_360_b200 as pkv
    from paged_kv_cache_360_b200.workloads import make_prefill_workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = make_prefill_workload(args.prefill_workload, seed=args.seed, rank=rank)
    slots, tables, lens = build_prefill_step(wl, library_pool(pkv))
    k, v = wl.k_cache.to(dev), wl.v_cache.to(dev)
    q, key, value = wl.q.to(dev), wl.new_key.to(dev), wl.new_value.to(dev)
    d_slots = torch.from_numpy(slots).to(dev)
    d_tables = torch.from_numpy(tables).to(dev)
    d_lens = torch.from_numpy(lens).to(dev)
    d_qs = torch.from_numpy(wl.query_start).to(dev)
    out = torch.empty_like(q)
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def append():
        pkv.paged_kv_append(k, v, key, value, d_slots, err_flag=err)

    def attend():
        pkv.paged_attention_prefill(out, q, k, v, d_tables, d_lens, d_qs, wl.scale, err_flag=err)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        n0 = pkv.launch_count()
        append()
        attend()
        launches_per_step = pkv.launch_count() - n0
    torch.cuda.synchronize()
    g_step, g_attn = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        append()
        attend()
    with torch.cuda.graph(g_attn, stream=stream):
        attend()
    torch.cuda.synchronize()
    flops = prefill_flops(lens, wl.query_start, wl.num_heads, wl.head_dim)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    def timed(graph, steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(steps):
                graph.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return e0.elapsed_time(e1)

    sampler = ClockSampler()
    if rank == 0:
        sampler.start()
        time.sleep(0.3)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_step.replay()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    step_ms = timed(g_step, args.steps)
    t_wall1 = time.time()
    attn_ms = timed(g_attn, args.steps)

    # end to end: pinned host inputs -> device, append + prefill, output -> pinned host
    h_in = [t.pin_memory() for t in (wl.q, wl.new_key, wl.new_value, torch.from_numpy(slots),
                                     torch.from_numpy(tables), torch.from_numpy(lens),
                                     torch.from_numpy(wl.query_start))]
    d_in = [torch.empty_like(t, device=dev) for t in h_in]
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    e2e_out = torch.empty_like(out)

    def e2e_step():
        for h, d in zip(h_in, d_in):
            d.copy_(h, non_blocking=True)
        pkv.paged_kv_append(k, v, d_in[1], d_in[2], d_in[3], err_flag=err)
        pkv.paged_attention_prefill(e2e_out, d_in[0], k, v, d_in[4], d_in[5], d_in[6], wl.scale,
                                    err_flag=err)
        h_out.copy_(e2e_out, non_blocking=True)

    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=stream):
        e2e_step()
    torch.cuda.synchronize()
    e2e_steps = max(3, min(args.steps, 500))
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            g_e2e.replay()
    e2e_ms = timed(g_e2e, e2e_steps)
    if rank == 0:
        sampler.stop()
    torch.cuda.synchronize()
    err_val = int(err.item())
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = h_out.numel() * h_out.element_size()

    step_ms, attn_ms, e2e_ms = max_over_ranks([step_ms, attn_ms, e2e_ms], world, dev)
    if rank != 0:
        return None
    peak, peak_sustained, peak_kind = measured_tensor_peak()
    ms_per_step = step_ms / args.steps
    attn_avg = attn_ms / args.steps
    achieved = flops / (attn_avg * 1e-3) / 1e12
    value = world * flops / (ms_per_step * 1e-3) / 1e12
    e2e_per_step = e2e_ms / e2e_steps
    nq = np.diff(wl.query_start)
    line = {
        "metric": PREFILL_METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == torch.bfloat16 else "f16",
        "data": "synthetic",
        "config": {"workload": wl.name, "num_seqs_per_gpu": wl.num_seqs,
                   "query_tokens_per_gpu": wl.num_tokens, "num_heads": wl.num_heads,
                   "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                   "block_size": wl.block_size, "num_blocks": wl.num_blocks,
                   "context_lens": [int(x) for x in lens],
                   "query_counts": [int(x) for x in nq], "seed": args.seed,
                   "parallelism": f"dp{world} (independent batches per GPU)",
                   "l2": "not flushed: the pool is %.0f MB, %.1fx the 126 MB L2"
                         % (2 * k.numel() * k.element_size() / 1e6,
                            2 * k.numel() * k.element_size() / 126e6),
                   "timing": "CUDA events around K back-to-back replays of the step's CUDA graph "
                             "(paged_kv_append of the query tokens' K/V, then the prefill)"},
        "attention_flops_per_step": flops,
        "roofline": {"bound": "tensor", "kernel": "paged_attention_prefill (tcgen05)",
                     "timing": "CUDA events around K back-to-back prefill-only graph replays",
                     "achieved": round(achieved, 2), "peak": peak,
                     "peak_kind": f"{peak_kind} bf16 dense burst",
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "frac_of_sustained": round(achieved / peak_sustained, 4) if peak_sustained else None,
                     "traffic": read_record("prefill_traffic.txt", prefill_device_sha256()),
                     "algorithmic_flops_per_launch": flops,
                     "avg_launch_ms": round(attn_avg, 5)},
        "e2e": {"value": round(world * flops / (e2e_per_step * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_per_step, 5), "steps": e2e_steps,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "path": "per step: pinned host -> device copies of q, the new K/V, slots, tables, "
                        "lengths and query starts; paged_kv_append; paged_attention_prefill; "
                        "device -> pinned host copy of the output; one stream, one CUDA graph"},
        "gpu_launches": int(launches_per_step * args.steps),
        "launches_per_step": int(launches_per_step),
        "device_err_flag": err_val,
        "clocks": sampler.summary(t_wall0, t_wall1),
    }
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = prefill_cpu_baseline(wl, slots, tables, lens, args.cpu_budget)
    return line


def prefill_cpu_baseline(wl, slots, tables, lens, budget_s):
    """The oracle's append + prefill on a bounded sample: the last m query
    tokens of the first chunked request (the prefill of a chunk of m tokens),
    m grown until about `budget_s` of CPU time."""
    import oracle
    oracle.build()
    nq = np.diff(wl.query_start)
    b = 1 if wl.num_seqs > 1 else 0
    L = int(lens[b])
    kw, vw = oracle.words(wl.k_cache), oracle.words(wl.v_cache)
    r0, r1 = int(wl.query_start[b]), int(wl.query_start[b + 1])
    oracle.append(kw, vw, wl.new_key[r0:r1], wl.new_value[r0:r1], slots[r0:r1])

    def sample(m):
        qs = np.array([0, m], dtype=np.int32)
        t0 = time.perf_counter()
        oracle.paged_prefill(wl.q[r1 - m:r1], kw, vw, tables[b:b + 1], lens[b:b + 1], qs, wl.scale)
        return time.perf_counter() - t0

    m = 1
    dt = sample(m)
    while m < int(nq[b]) and dt * 2 < budget_s:
        m = min(int(nq[b]), m * 2)
        dt = sample(m)
    fl = prefill_flops([L], [0, m], wl.num_heads, wl.head_dim)
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
            "seconds": round(dt, 3),
            "sample": f"oracle prefill of the last {m} query tokens of request {b} "
                      f"(context {L}) of the {wl.name} batch, single-threaded C float64"}


# ------------------------------------------------------ CPU oracle (baseline)

def sample_bytes(wl, sub_lens, n) -> int:
    """Algorithmic bytes of an oracle sample: n whole sequences decoded (plus
    their appended tokens when the workload appends one per sequence)."""
    es = 2
    sub = np.asarray(sub_lens, dtype=np.int64)
    return int(sub.sum()) * wl.num_kv_heads * wl.head_dim * es * 2 + \
        2 * n * wl.num_heads * wl.head_dim * es + \
        int(np.sum((sub + wl.block_size - 1) // wl.block_size)) * 4 + 4 * n + \
        (0 if wl.prefix_len else append_bytes(n, wl))


def _oracle_sample(wl, tables, lens, slots, key, value, seqs):
    """Oracle append of the sample's new tokens, then oracle decode of the sample."""
    import oracle
    kw, vw = oracle.words(wl.k_cache), oracle.words(wl.v_cache)
    if not wl.prefix_len:
        idx = np.asarray(seqs)
        oracle.append(kw, vw, key[idx], value[idx], slots[idx])
    t = np.ascontiguousarray(tables[seqs])
    l = np.ascontiguousarray(lens[seqs])
    return oracle.paged_decode(wl.q[seqs], kw, vw, t, l, wl.scale)


def cpu_baseline(wl, lens, tables, slots, key, value, budget_s=12.0):
    """Time the oracle (single-threaded C, float64) on a bounded sample: whole
    sequences of the same batch, in order, until about `budget_s` of CPU time."""
    import oracle
    oracle.build()
    # calibrate on the first sequence
    t0 = time.perf_counter()
    _oracle_sample(wl, tables, lens, slots, key, value, [0])
    per_token = (time.perf_counter() - t0) / max(1, int(lens[0]))
    n, tokens = 0, 0
    while n < wl.num_seqs and (tokens + int(lens[n])) * per_token < budget_s:
        tokens += int(lens[n])
        n += 1
    n = max(n, 1)
    seqs = list(range(n))
    t0 = time.perf_counter()
    _oracle_sample(wl, tables, lens, slots, key, value, seqs)
    dt = time.perf_counter() - t0
    sub_lens = lens[:n]
    nbytes = sample_bytes(wl, sub_lens, n)
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "seconds": round(dt, 3), "sample_seqs": n,
            "seq_decode_steps_per_s": round(n / dt, 3),
            "sample": f"first {n} of {wl.num_seqs} sequences of the {wl.name} batch "
                      f"({int(np.sum(sub_lens))} context tokens): oracle append + decode, 1 pass, "
                      f"single-threaded C float64 on {os.cpu_count()} host cores available"}


def _oracle_worker(config, seed, seqs, barrier, results):
    """Spawned process: rebuild the same batch and step bookkeeping (the
    generator is a pure function of the seed), wait for the others, then time
    the oracle on its share of the sample."""
    from paged_kv_cache_360_b200.workloads import make_workload
    import oracle
    oracle.build()
    wl = make_workload(config, seed=seed, rank=0)
    pairs, slots, tables, lens, key, value = build_step(wl, oracle_pool())
    barrier.wait()
    t0 = time.perf_counter()
    _oracle_sample(wl, tables, lens, slots, key, value, seqs)
    results.put(time.perf_counter() - t0)


def cpu_baseline_all_cores(wl, lens, n, max_workers=32):
    """The same sample as cpu_baseline (the first n sequences), shared out over
    one spawned process per host core (greedy by length), all starting
    together; throughput = the sample's bytes / the slowest process's time."""
    import multiprocessing as mp
    workers = max(1, min(os.cpu_count() or 1, n, max_workers))
    shares = [[] for _ in range(workers)]
    loads = [0] * workers
    for b in sorted(range(n), key=lambda b: -int(lens[b])):
        w = loads.index(min(loads))
        shares[w].append(b)
        loads[w] += int(lens[b])
    ctx = mp.get_context("spawn")
    barrier, results = ctx.Barrier(workers), ctx.Queue()
    procs = [ctx.Process(target=_oracle_worker, args=(wl.config, wl.seed, sorted(sh), barrier, results))
             for sh in shares]
    for pr in procs:
        pr.start()
    import queue as _queue
    times, deadline = [], time.time() + 900
    try:
        while len(times) < workers:
            try:
                times.append(results.get(timeout=5))
            except _queue.Empty:
                if time.time() > deadline or any(pr.exitcode not in (None, 0) for pr in procs):
                    raise RuntimeError("an oracle process failed or ran past its limit")
    finally:
        for pr in procs:
            pr.join(timeout=30)
            if pr.is_alive():
                pr.terminate()
    dt = max(times)
    nbytes = sample_bytes(wl, lens[:n], n)
    return {"value": round(nbytes / dt / 1e9, 4), "cores": workers, "seconds": round(dt, 3)}


def run_reference_prefill(args, rank, world):
    """The oracle as the reference arm of the prefill step: each step is the
    oracle's append + prefill of the last m query tokens of the first chunked
    request, m sized so that a step takes about --ref-step-budget seconds."""
    if rank != 0:
        return None
    from paged_kv_cache_360_b200.workloads import make_prefill_workload
    import oracle
    oracle.build()
    wl = make_prefill_workload(args.prefill_workload, seed=args.seed, rank=0)
    slots, tables, lens = build_prefill_step(wl, oracle_pool())
    b = 1 if wl.num_seqs > 1 else 0
    r0, r1 = int(wl.query_start[b]), int(wl.query_start[b + 1])
    kw, vw = oracle.words(wl.k_cache), oracle.words(wl.v_cache)

    def step(m):
        t0 = time.perf_counter()
        oracle.append(kw, vw, wl.new_key[r1 - m:r1], wl.new_value[r1 - m:r1], slots[r1 - m:r1])
        oracle.paged_prefill(wl.q[r1 - m:r1], kw, vw, tables[b:b + 1], lens[b:b + 1],
                             np.array([0, m], dtype=np.int32), wl.scale)
        return time.perf_counter() - t0

    m = 1
    dt = step(m)
    while m < r1 - r0 and dt * 2 < args.ref_step_budget:
        m = min(r1 - r0, m * 2)
        dt = step(m)
    for _ in range(args.warmup):
        step(m)
    total = sum(step(m) for _ in range(args.steps))
    ms = total / args.steps * 1e3
    fl = prefill_flops([int(lens[b])], [0, m], wl.num_heads, wl.head_dim)
    tf = fl / (ms * 1e-3) / 1e12
    sample = (f"each step: oracle append + prefill of the last {m} query tokens of request {b} "
              f"(context {int(lens[b])}) of the {wl.name} batch, single-threaded C float64")
    return {"impl": "reference", "metric": PREFILL_METRIC, "value": round(tf, 6), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "query_tokens_sampled": m, "num_heads": wl.num_heads,
                       "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                       "block_size": wl.block_size, "seed": args.seed},
            "cpu_baseline": {"value": round(tf, 6), "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(tf, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    from paged_kv_cache_360_b200.workloads import make_workload
    import oracle
    oracle.build()
    wl = make_workload(args.config, seed=args.seed, rank=0)
    pairs, slots, tables, lens, key, value = build_step(wl, oracle_pool())
    budget = args.ref_step_budget
    t0 = time.perf_counter()
    _oracle_sample(wl, tables, lens, slots, key, value, [0])
    per_token = (time.perf_counter() - t0) / max(1, int(lens[0]))
    n, tokens = 0, 0
    while n < wl.num_seqs and (tokens + int(lens[n])) * per_token < budget:
        tokens += int(lens[n])
        n += 1
    n = max(n, 1)
    seqs = list(range(n))
    for _ in range(args.warmup):
        _oracle_sample(wl, tables, lens, slots, key, value, seqs)
    total = 0.0
    for _ in range(args.steps):
        t0 = time.perf_counter()
        _oracle_sample(wl, tables, lens, slots, key, value, seqs)
        total += time.perf_counter() - t0
    sub_lens = lens[:n]
    nbytes = sample_bytes(wl, sub_lens, n)
    ms = total / args.steps * 1e3
    value_gbs = nbytes / (ms * 1e-3) / 1e9
    sample = (f"each step: first {n} of {wl.num_seqs} sequences of the {wl.name} batch "
              f"({int(np.sum(sub_lens))} context tokens), oracle append + decode, single-threaded C float64")
    return {"impl": "reference", "metric": METRIC, "value": round(value_gbs, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "num_seqs_sampled": n, "num_heads": wl.num_heads,
                       "num_kv_heads": wl.num_kv_heads, "head_dim": wl.head_dim,
                       "block_size": wl.block_size, "seed": args.seed},
            "seq_decode_steps_per_s": round(n / (ms * 1e-3), 3),
            "cpu_baseline": {"value": round(value_gbs, 4), "unit": "GB/s", "cores": 1,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value_gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--config", type=int, default=2, choices=[1, 2, 3, 4, 5])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--partition-size", type=int, default=None,
                    help="0 = balanced split (default unless the workload fixes one); "
                         "> 0 = fixed partitions of that many tokens")
    ap.add_argument("--shared-prefix", action="store_true",
                    help="decode through paged_attention_decode_shared_prefix (workloads with a "
                         "shared prompt prefix: --config 3)")
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "prefill"], default="decode",
                    help="decode: the decode step (default); prefill: the paged prefill step")
    ap.add_argument("--prefill-workload", default="prefill-llama3-8b-layer")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the extra records (prefill, decode on the other workloads, "
                         "data-movement kernels) of the decode line")
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle CPU time")
    ap.add_argument("--ref-step-budget", type=float, default=3.0,
                    help="seconds of oracle CPU time per reference step")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            ap.error("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    if args.impl == "reference":
        line = (run_reference_prefill if args.workload == "prefill" else run_reference)(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        run = run_prefill if args.workload == "prefill" else run_ours
        line = run(args, rank, world, local_rank)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
