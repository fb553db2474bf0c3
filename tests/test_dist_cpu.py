"""Multi-rank host logic of bench.py, on CPU with the gloo backend (world size 2).

The benchmark shards nothing across ranks (each GPU runs its own copy of the
workload); what must hold across ranks is the timing: every rank takes the same
collective steps and the reported time is the maximum over ranks.
"""

import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, local = bench.dist_env()
        assert (r, w, local) == (rank, world, rank)
        bench.barrier(world)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        bench.barrier(world)
        # the reference arm: ranks other than 0 exit without work or output
        class A:
            steps, warmup = 1, 3
        ref = bench.run_reference(A, rank, world) if rank != 0 else None
        out[rank] = (t, ref)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_barrier_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == pytest.approx(15.0)
    assert res[1][0] == pytest.approx(15.0)
    assert res[1][1] is None


def test_single_rank_identity():
    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks(3.25, 1) == 3.25
    bench.barrier(1)  # no process group needed for one rank


def test_flop_convention():
    sys.path.insert(0, ROOT)
    import bench

    # forward = 4 B H N^2 d, halved when causal; backward = 2.5x forward
    assert bench.fwd_flops(2, 32, 8192, 128, True) == 4 * 2 * 32 * 8192 ** 2 * 128 / 2
    assert bench.fwd_flops(1, 1, 10, 64, False) == 4 * 100 * 64
    assert bench.bwd_flops(2, 32, 8192, 128, True) == 2.5 * bench.fwd_flops(2, 32, 8192, 128, True)
