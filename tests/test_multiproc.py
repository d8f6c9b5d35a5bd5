"""The multi-GPU bench path runs one independent replica per rank (weak scaling); its only
collective is the max-over-ranks step time. This checks that reduction and the whole-job
throughput formula with two gloo ranks on CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms = 10.0 + 5.0 * rank  # the slower rank sets the step time
        got = bench.max_over_ranks(ms, world)
        dist.barrier()
        out[rank] = (got, bench.aggregate_tflops(world, 6.594e12, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_aggregate_gloo_two_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # two replicas, each 6.594e12 FLOP per 15 ms step
    assert res[0][1] == pytest.approx(2 * 6.594e12 / 15e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate_tflops(1, 1e12, 1.0) == pytest.approx(1000.0)
