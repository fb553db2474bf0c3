"""Host logic of the sequence-sharded forward and backward (striped tokens, K/V ring) on CPU.

The ring schedule, the diagonal offsets and the point-to-point exchanges of
``exact_io_aware_61_b200.seqpar.ring_forward`` and ``ring_backward`` run here
over gloo ranks, with the fp64 oracle standing in for the CUDA calls (block
forward and merge; preprocess, block backward, dQ conversion); the gathered
results must equal the oracle's attention and gradients over the whole,
unsharded sequence. The CUDA calls themselves are checked on the GPU.
"""

import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle.attention as ORACLE  # noqa: E402
from exact_io_aware_61_b200 import inputs as INP  # noqa: E402
from exact_io_aware_61_b200 import seqpar  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_block(q, k, v, o, lse, causal, scale, diag_offset):
    """The block forward as fa_fwd_partial defines it: row i sees key j iff j <= i + diag_offset."""
    n = q.shape[2]
    bo, bl = ORACLE.attention_forward_positions(q.numpy(), k.numpy(), v.numpy(), np.arange(n) + diag_offset,
                                                np.arange(n), scale, causal)
    o.copy_(torch.from_numpy(bo))
    lse.copy_(torch.from_numpy(bl))


def oracle_merge(o_parts, lse_parts, o, lse):
    P, d = o_parts.shape[0], o_parts.shape[-1]
    mo, ml = ORACLE.merge_outputs(o_parts.reshape(P, -1, d).numpy(), lse_parts.reshape(P, -1).double().numpy())
    o.copy_(torch.from_numpy(mo).view_as(o))
    lse.copy_(torch.from_numpy(ml).view_as(lse))


SHAPE = dict(B=2, Hq=4, Hkv=2, N=24, d=8)


def _ring_worker(rank, world, port, causal, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = INP.make_inputs(SHAPE["B"], SHAPE["Hq"], SHAPE["Hkv"], SHAPE["N"], SHAPE["d"], "f32", seed=131)
        q, k, v = (inp[n].double() for n in ("q", "k", "v"))
        shards = [seqpar.shard_striped(t, rank, world) for t in (q, k, v)]
        o, lse = seqpar.ring_forward(*shards, causal=causal, scale=0.37, block=oracle_block, merge=oracle_merge)
        out[rank] = (o.numpy().tolist(), lse.numpy().tolist())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_forward_equals_unsharded_attention_gloo(world, causal):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_ring_worker, args=(world, port, causal, out), nprocs=world, join=True)
        res = dict(out)
    inp = INP.make_inputs(SHAPE["B"], SHAPE["Hq"], SHAPE["Hkv"], SHAPE["N"], SHAPE["d"], "f32", seed=131)
    q, k, v = (INP.as_f64(inp[n]) for n in ("q", "k", "v"))
    want_o, want_lse = ORACLE.attention_forward(q, k, v, 0.37, causal)
    got_o = seqpar.unshard_striped([torch.tensor(res[r][0]) for r in range(world)]).numpy()
    got_lse = seqpar.unshard_striped([torch.tensor(res[r][1])[..., None] for r in range(world)])[..., 0].numpy()
    # LSE travels in float32 (the library's type); the merge weights carry its rounding
    assert np.max(np.abs(got_lse - want_lse)) < 1e-5
    assert np.max(np.abs(got_o - want_o)) < 1e-5


def test_ring_schedule_visits_every_rank_once_with_the_striped_diagonal():
    for world in (1, 2, 3, 8):
        for rank in range(world):
            sched = seqpar.ring_schedule(rank, world, True)
            assert sorted(s for s, _ in sched) == list(range(world))
            assert sched[0] == (rank, 0)  # the local block first: nothing to wait for
            for src, diag in sched:
                # local row i is position i*W + rank, key row j is j*W + src:
                # visible iff j*W + src <= i*W + rank iff j <= i + diag
                W = world
                for i in range(4):
                    for j in range(4):
                        assert (j * W + src <= i * W + rank) == (j <= i + diag)
            assert all(d == 0 for _, d in seqpar.ring_schedule(rank, world, False))


def test_striped_shards_round_trip():
    x = torch.arange(2 * 3 * 12 * 4).reshape(2, 3, 12, 4)
    shards = [seqpar.shard_striped(x, r, 4) for r in range(4)]
    assert all(s.is_contiguous() and s.shape == (2, 3, 3, 4) for s in shards)
    assert torch.equal(shards[1][:, :, 2], x[:, :, 9])
    assert torch.equal(seqpar.unshard_striped(shards), x)
    assert torch.equal(seqpar.striped_positions(3, 1, 4), torch.tensor([1, 5, 9]))
    with pytest.raises(ValueError):
        seqpar.shard_striped(x, 0, 5)


class OracleBackwardOps:
    """The fp64 oracle in place of fa_bwd_prep / fa_bwd_partial / fa_bwd_dq / fa_f32_to_bf16."""

    def __init__(self, causal, scale):
        self.causal, self.scale = causal, scale

    def prep(self, o, lse, do):
        self.lse = lse.double().numpy()
        self.D = np.sum(do.double().numpy() * o.double().numpy(), axis=-1)
        self.dq = None

    def block(self, q, k, v, do, dk_acc, dv_acc, diag_offset):
        n = q.shape[2]
        bq, bk, bv = ORACLE.attention_backward_block(q.numpy(), k.numpy(), v.numpy(), do.numpy(), self.lse, self.D,
                                                     np.arange(n) + diag_offset, np.arange(n), self.scale, self.causal)
        self.dq = bq if self.dq is None else self.dq + bq
        dk_acc += torch.from_numpy(bk).to(dk_acc.dtype)
        dv_acc += torch.from_numpy(bv).to(dv_acc.dtype)

    def finish(self, dq):
        dq.copy_(torch.from_numpy(self.dq))

    def to_bf16(self, src, dst):
        dst.copy_(src)


def _ring_bwd_worker(rank, world, port, causal, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = INP.make_inputs(SHAPE["B"], SHAPE["Hq"], SHAPE["Hkv"], SHAPE["N"], SHAPE["d"], "f32", seed=137,
                              grad=True)
        q, k, v, do = (inp[n].double() for n in ("q", "k", "v", "do"))
        o, lse = ORACLE.attention_forward(q.numpy(), k.numpy(), v.numpy(), 0.37, causal)
        sh = lambda t: seqpar.shard_striped(t, rank, world)
        # the dK/dV accumulators are f32, as the library's; dQ and the exchange of K, V in f64
        o_r = sh(torch.from_numpy(o))
        lse_r = sh(torch.from_numpy(lse)[..., None])[..., 0]
        dq, dk, dv = seqpar.ring_backward(sh(q), sh(k), sh(v), o_r, lse_r, sh(do), causal=causal, scale=0.37,
                                          ops=OracleBackwardOps(causal, 0.37))
        out[rank] = tuple(t.numpy().tolist() for t in (dq, dk, dv))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [True, False])
def test_ring_backward_equals_unsharded_gradients_gloo(world, causal):
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_ring_bwd_worker, args=(world, port, causal, out), nprocs=world, join=True)
        res = dict(out)
    inp = INP.make_inputs(SHAPE["B"], SHAPE["Hq"], SHAPE["Hkv"], SHAPE["N"], SHAPE["d"], "f32", seed=137, grad=True)
    q, k, v, do = (INP.as_f64(inp[n]) for n in ("q", "k", "v", "do"))
    rq, rk, rv, _ = ORACLE.attention_backward(q, k, v, do, 0.37, causal)
    for i, ref in enumerate((rq, rk, rv)):
        got = seqpar.unshard_striped([torch.tensor(res[r][i]) for r in range(world)]).numpy()
        # dK, dV accumulate in float32 across the ring
        assert np.max(np.abs(got - ref)) < 1e-5 * max(1.0, np.max(np.abs(ref)))
