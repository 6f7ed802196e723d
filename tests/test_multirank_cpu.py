"""The multi-rank plumbing of bench.py, run as two gloo ranks on the CPU.

Sequences never interact in the layer, so N ranks run N independent batches with no exchange on
the path; what the ranks share is the accounting: the job's time is the slowest rank's and its work
the sum of the ranks' tokens.  The reference leg runs on rank 0 alone.
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


def _worker(rank: int, world: int, port: int, q):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        # ranks report different times and different token counts
        ms, tokens = bench.combine_over_ranks(10.0 + 5.0 * rank, 1000 + rank, world, "cpu")
        # a second call in the same order must see the same combined values on every rank
        ms2, tokens2 = bench.combine_over_ranks(3.0 * (world - rank), 7, world, "cpu")

        class Args:
            workload, steps, warmup = "tiny_fp32", 1, 1
        ref = bench.run_reference(Args(), rank, world) if rank != 0 else "skipped"
        q.put((rank, ms, tokens, ms2, tokens2, ref))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_combine_time_and_tokens():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    results.sort()
    for rank, ms, tokens, ms2, tokens2, ref in results:
        assert ms == 15.0 and tokens == 2001            # max of 10, 15; sum of 1000, 1001
        assert ms2 == 6.0 and tokens2 == 14             # max of 6, 3; sum of 7, 7
        if rank != 0:
            assert ref is None                           # the reference leg runs on rank 0 only


def test_single_rank_combination_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.combine_over_ranks(2.5, 11, 1, "cpu") == (2.5, 11)
