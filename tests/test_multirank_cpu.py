"""The multi-rank path of bench.py on CPU: two gloo ranks, max-over-ranks timing and weak-scaling
throughput.  The decode path partitions by sequence, so ranks exchange only these timing scalars."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        ms = 10.0 + 5.0 * rank                        # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, dist, torch.device("cpu"))
        out[rank] = (worst, bench.job_throughput(world, 1e9, worst))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0
    # two ranks each moving 1 GB per step, slowest step 15 ms -> 2 GB / 15 ms
    assert abs(res[0][1] - 2e9 / 15e-3 / 1e9) < 1e-9


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert abs(bench.job_throughput(1, 193257984 * 96, 15.6) - 1189.3) < 1.0


def test_profile_hash_ignores_comments_only():
    """A committed ncu summary stays valid across comment edits of the kernel sources, not code edits."""
    sys.path.insert(0, ROOT)
    import bench
    a = b"int x = 1; // old note\n/* block\n comment */ float y;\n"
    assert bench._code_only(a) == bench._code_only(b"int x = 1;   // new note\nfloat y;")
    assert bench._code_only(a) != bench._code_only(b"int x = 2; float y;")
