"""The N>1 host logic of bench.py on CPU: two gloo ranks in spawned processes.

Per-rank seeds differ (each replica streams its own batch, no collective on the
data path), timings are reduced with a max over ranks, and the whole-job value
counts every rank's bytes against the slowest rank's time.
"""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    sys.path.insert(0, ROOT)
    import bench
    from paged_kv_cache_418_b200 import workloads as W
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms, dec = bench.max_over_ranks([10.0 + 3 * rank, 7.0 - rank], world, torch.device("cpu"))
        seed = bench.rank_seed(3, rank)
        w = W.shrink_workload(3, seed=seed, B=2, max_ctx=64)
        dist.barrier()
        q.put((rank, ms, dec, seed, int(w.context_lens.sum()), float(w.q.reshape(-1)[:8].sum())))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_own_batches():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(world):
            r, ms, dec, seed, ctx_sum, qsum = q.get(timeout=120)
            got[r] = (ms, dec, seed, ctx_sum, qsum)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    # max over ranks, elementwise, seen identically by both ranks
    assert got[0][:2] == got[1][:2] == (13.0, 7.0)
    # each replica has its own seed and therefore its own batch
    assert got[0][2] != got[1][2]
    assert got[0][3:] != got[1][3:]


def test_job_value_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_value(10**9, 100, 1, 50.0)
    two = bench.job_value(10**9, 100, 2, 50.0)
    assert two == pytest.approx(2 * one)
    assert one == pytest.approx(10**9 * 100 / 0.05 / 1e9)
    assert bench.max_over_ranks([1.5, 2.5], 1, None) == [1.5, 2.5]
