"""The multi-GPU bench path on CPU: two gloo ranks (no GPU).

Each rank draws its own batch (the rank keys the seed), the device times are
reduced with a max over ranks, and the whole-job throughput counts every rank's
bytes against the slowest rank's time."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from paged_kv_cache_360_b200.workloads import make_workload
        wl = make_workload(2, seed=0, rank=rank, materialize=False)
        times = bench.max_over_ranks([1.0 + rank, 5.0 - rank], world)
        dist.barrier()
        out[rank] = (times, wl.context_lens.tolist(), wl.free_order[:16].tolist(), wl.num_seqs)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_take_the_max():
    world = 2
    with mp.Manager() as manager:
        out = manager.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == [2.0, 5.0]
    assert res[0][1] != res[1][1] and res[0][2] != res[1][2]      # independent batches
    assert res[0][3] == res[1][3] == 64                            # same per-rank batch size
    import bench
    assert bench.whole_job_gbs(1e9, 2, 1.0) == 2 * bench.whole_job_gbs(1e9, 1, 1.0)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
