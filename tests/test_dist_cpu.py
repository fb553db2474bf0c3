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


# ------------------------------------------- (batch, KV head) partition

def test_pair_range_covers_every_pair_once():
    sys.path.insert(0, ROOT)
    from exact_io_aware_61_b200.shard import pair_range

    for B, Hq, Hkv in ((2, 32, 32), (1, 32, 8), (3, 6, 3), (1, 4, 1), (5, 8, 2)):
        for world in (1, 2, 3, 4, 8, 16):
            seen = []
            sizes = []
            for r in range(world):
                s = pair_range(B, Hq, Hkv, r, world)
                seen.extend(range(s.p0, s.p1))
                sizes.append(s.pairs)
                lb, lq, lkv = s.local_shape()
                assert lb * lkv == s.pairs and lq == lkv * (Hq // Hkv)
            assert seen == list(range(B * Hkv))          # contiguous, disjoint, complete, in rank order
            assert max(sizes) - min(sizes) <= 1          # balanced


def _shard_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import numpy as np
    import torch

    import oracle.attention as ORACLE
    from exact_io_aware_61_b200 import inputs as INP
    from exact_io_aware_61_b200.shard import kv_view, pair_range, q_view

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, N, d = 3, 4, 2, 37, 8
        inp = INP.make_inputs(B, Hq, Hkv, N, d, "f32", seed=77, grad=True)
        g = {n: t.double() for n, t in inp.items()}
        s = pair_range(B, Hq, Hkv, rank, world)
        # this rank's problem: views of its slice, B = 1
        q, do = q_view(g["q"], s), q_view(g["do"], s)
        k, v = kv_view(g["k"], s), kv_view(g["v"], s)
        o, lse = ORACLE.attention_forward(q.numpy(), k.numpy(), v.numpy(), 0.3, True)
        dq, dk, dv, _ = ORACLE.attention_backward(q.numpy(), k.numpy(), v.numpy(), do.numpy(), 0.3, True)
        # reassemble on every rank: all-gather the slices (ranks hold different sizes, so pad to the largest)
        pieces = {}
        for name, arr, per in (("o", o, Hq // Hkv), ("lse", lse, Hq // Hkv), ("dq", dq, Hq // Hkv),
                               ("dk", dk, 1), ("dv", dv, 1)):
            t = torch.from_numpy(np.ascontiguousarray(arr.reshape(arr.shape[0] * arr.shape[1], *arr.shape[2:])))
            most = -(-B * Hkv // world) * per
            pad = torch.zeros((most,) + tuple(t.shape[1:]), dtype=t.dtype)
            pad[:t.shape[0]] = t
            bufs = [torch.zeros_like(pad) for _ in range(world)]
            dist.all_gather(bufs, pad)
            parts = []
            for r in range(world):
                sr = pair_range(B, Hq, Hkv, r, world)
                parts.append(bufs[r][:sr.pairs * per])
            pieces[name] = torch.cat(parts).numpy()
        out[rank] = {n: a.tolist() for n, a in pieces.items()}
    finally:
        dist.destroy_process_group()


def test_pair_shards_reassemble_into_the_single_rank_result_gloo():
    """Two gloo ranks each run the fp64 oracle on their slice of (batch, KV
    head) pairs through the shard views, gather the slices, and the result
    equals the oracle on the whole problem: the partition needs no exchange
    beyond collecting the outputs."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import oracle.attention as ORACLE
    from exact_io_aware_61_b200 import inputs as INP

    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_shard_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    B, Hq, Hkv, N, d = 3, 4, 2, 37, 8
    inp = INP.make_inputs(B, Hq, Hkv, N, d, "f32", seed=77, grad=True)
    q, k, v, do = (INP.as_f64(inp[n]) for n in ("q", "k", "v", "do"))
    o, lse = ORACLE.attention_forward(q, k, v, 0.3, True)
    dq, dk, dv, _ = ORACLE.attention_backward(q, k, v, do, 0.3, True)
    want = {"o": o.reshape(B * Hq, N, d), "lse": lse.reshape(B * Hq, N), "dq": dq.reshape(B * Hq, N, d),
            "dk": dk.reshape(B * Hkv, N, d), "dv": dv.reshape(B * Hkv, N, d)}
    for rank in range(world):
        for name, ref in want.items():
            got = np.asarray(res[rank][name])
            assert got.shape == ref.shape, (name, got.shape)
            assert np.max(np.abs(got - ref)) < 1e-12, (rank, name)
