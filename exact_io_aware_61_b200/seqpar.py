"""Attention sharded over the sequence dimension: striped tokens, a ring of K/V, one merge.

The pages name parallelism over the sequence dimension (synthetic.wiki
"FlashAttention: attention's bottleneck is the wire, not the maths", section
"Versions, and what the numbers say") and give the rescale rule that makes a
merge of per-block softmax results exact (fanfani.net "FlashAttention",
section "A pinch of math: making the softmax work in pieces"). Sharding the
sequence across ``W`` ranks:

* **Striped assignment.** Token ``t`` of every sequence lives on rank
  ``t mod W``: rank ``r`` holds ``x[:, :, r::W]`` of Q, K and V as dense
  ``[B, H, N / W, d]`` tensors. Local row ``i`` of rank ``r`` is position
  ``i W + r``, so rank ``r``'s queries against rank ``c``'s keys form a causal
  block whose diagonal sits at offset 0 when ``c <= r`` (key ``j`` visible iff
  ``j <= i``) and at -1 when ``c > r`` (``j <= i - 1``). Every block holds
  about half of an ``n x n`` square, so under the causal mask every rank does
  the same work; a contiguous split would leave the last rank with ``W``
  times the work of the first.
* **Ring.** K and V travel round the ring of ranks, ``W - 1`` hops: at step
  ``t`` rank ``r`` holds the K/V of rank ``(r - t) mod W``, computes that block
  with ``fa_fwd_partial`` while the next hop's transfer is in flight, and
  keeps the block's normalised output and LSE.
* **Merge.** ``fa_merge_partials`` combines the ``W`` blocks of every query
  row with the rescale rule. Only K/V cross the links; Q, O and the partial
  results stay on their rank.
* **Backward.** The same ring. Each rank prepares its own rows once (D from
  its O and dO, the merged LSE of its whole rows). At each step it adds the
  visiting key block's share of dK and dV into f32 accumulators that travel
  with that block, and its share of dQ into the rank's own accumulator
  (``fa_bwd_partial``). After the last step the accumulators are back at the
  ranks that own the keys.

The exchange uses ``torch.distributed`` point-to-point operations (NCCL over
NVLink on GPUs; any backend for the host logic). Every step of the attention
arithmetic runs in the CUDA library; ``block`` and ``merge`` can be replaced
(tests drive the same schedule and exchange with other implementations).
"""

from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch
import torch.distributed as dist

from . import _lib


def striped_positions(n_local: int, rank: int, world: int) -> torch.Tensor:
    """Sequence positions of the ``n_local`` rows that rank ``rank`` holds."""
    return rank + world * torch.arange(n_local)


def shard_striped(x: torch.Tensor, rank: int, world: int) -> torch.Tensor:
    """Rank ``rank``'s rows of ``x [B, H, N, d]`` (``N`` a multiple of ``world``), contiguous."""
    if x.shape[2] % world:
        raise ValueError(f"sequence length {x.shape[2]} is not a multiple of {world} ranks")
    return x[:, :, rank::world].contiguous()


def unshard_striped(shards: List[torch.Tensor]) -> torch.Tensor:
    """Inverse of :func:`shard_striped`: interleave the ranks' rows (dimension 2) back into sequence order."""
    world = len(shards)
    first = shards[0]
    out = first.new_empty(first.shape[:2] + (first.shape[2] * world,) + first.shape[3:])
    for r, s in enumerate(shards):
        out[:, :, r::world] = s
    return out


def ring_schedule(rank: int, world: int, causal: bool) -> List[Tuple[int, int]]:
    """``(source rank, diagonal offset)`` of the K/V block rank ``rank`` computes at each ring step.

    At step ``t`` the K/V of rank ``(rank - t) mod world`` has arrived. Under
    the causal mask, a source at or before ``rank`` shares the diagonal
    (offset 0) and a later one sees strictly earlier tokens only (offset -1);
    without the mask the offset is unused (0).
    """
    out = []
    for t in range(world):
        src = (rank - t) % world
        out.append((src, 0 if (not causal or src <= rank) else -1))
    return out


BlockFn = Callable[..., None]
MergeFn = Callable[..., None]


def _library_block(q, k, v, o, lse, causal, scale, diag_offset, stream=None):
    _lib.fa_fwd_partial(q, k, v, o, lse, causal, scale, diag_offset, stream)


def _library_merge(o_parts, lse_parts, o, lse, stream=None):
    _lib.fa_merge_partials(o_parts, lse_parts, o, lse, stream)


def ring_forward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                 scale: Optional[float] = None, group=None, *, block: Optional[BlockFn] = None,
                 merge: Optional[MergeFn] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Forward of attention over a sequence striped across the ranks of ``group``.

    ``q [B, Hq, n, d]``, ``k``, ``v [B, Hkv, n, d]`` are this rank's striped
    shards (:func:`shard_striped`), the same ``n`` on every rank. Returns this
    rank's rows of ``(O, LSE)``: ``O [B, Hq, n, d]``, ``LSE [B, Hq, n]`` float32.
    Collective: every rank of ``group`` must call it with the same shapes.
    """
    block = block or _library_block
    merge = merge or _library_merge
    if scale is None:
        scale = q.shape[-1] ** -0.5
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    o = torch.empty_like(q)
    lse = torch.empty(q.shape[:-1], dtype=torch.float32, device=q.device)
    if world == 1:
        block(q, k, v, o, lse, causal, scale, 0)
        return o, lse
    nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
    prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
    o_parts = q.new_empty((world,) + tuple(q.shape))
    lse_parts = torch.empty((world,) + tuple(q.shape[:-1]), dtype=torch.float32, device=q.device)
    recv = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    cur_k, cur_v = k, v
    for t, (src, diag) in enumerate(ring_schedule(rank, world, causal)):
        reqs = []
        if t + 1 < world:
            nk, nv = recv[t % 2]
            # the receive buffer last held the block computed two steps ago;
            # the transfer is ordered after that computation on the stream
            reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, cur_k, nxt, group),
                dist.P2POp(dist.isend, cur_v, nxt, group),
                dist.P2POp(dist.irecv, nk, prv, group),
                dist.P2POp(dist.irecv, nv, prv, group),
            ])
        block(q, cur_k, cur_v, o_parts[t], lse_parts[t], causal, scale, diag)
        for req in reqs:
            req.wait()
        if t + 1 < world:
            cur_k, cur_v = recv[t % 2]
    merge(o_parts, lse_parts, o, lse)
    return o, lse


class LibraryBackwardOps:
    """The CUDA calls of :func:`ring_backward` for one rank: ``fa_bwd_prep``,
    ``fa_bwd_partial`` per key block, ``fa_bwd_dq``, ``fa_f32_to_bf16``."""

    def __init__(self, q, k, causal: bool, scale: float, stream=None):
        B, Hq, n, d = q.shape
        self.Hkv = k.shape[1]
        self.causal, self.scale, self.stream = causal, scale, stream
        self.ws = torch.empty(max(_lib.fa_bwd_workspace_size(B, Hq, self.Hkv, n, d), 16), dtype=torch.uint8,
                              device=q.device)

    def prep(self, o, lse, do):
        _lib.fa_bwd_prep(o, lse, do, self.ws, self.Hkv, self.stream)

    def block(self, q, k, v, do, dk_acc, dv_acc, diag_offset: int):
        _lib.fa_bwd_partial(q, k, v, do, dk_acc, dv_acc, self.ws, self.causal, self.scale, diag_offset, self.stream)

    def finish(self, dq):
        _lib.fa_bwd_dq(dq, self.ws, self.Hkv, self.stream)

    def to_bf16(self, src, dst):
        _lib.fa_f32_to_bf16(src, dst, self.stream)


def ring_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, lse: torch.Tensor,
                  do: torch.Tensor, causal: bool = False, scale: Optional[float] = None, group=None, *,
                  ops=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients of :func:`ring_forward` for this rank's striped shards.

    ``o`` and ``lse`` are this rank's rows of the forward (``ring_forward``'s
    results: the merged, whole-row values), ``do`` the upstream gradient of
    ``o``. Returns this rank's rows of ``(dQ, dK, dV)``, shaped like ``q``,
    ``k``, ``v``. Collective over ``group``, like :func:`ring_forward`.
    """
    if scale is None:
        scale = q.shape[-1] ** -0.5
    ops = ops or LibraryBackwardOps(q, k, causal, scale)
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    ops.prep(o, lse, do)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    acc = (torch.zeros(k.shape, dtype=torch.float32, device=k.device),
           torch.zeros(v.shape, dtype=torch.float32, device=v.device))
    if world == 1:
        ops.block(q, k, v, do, acc[0], acc[1], 0)
    else:
        nxt = dist.get_global_rank(group, (rank + 1) % world) if group is not None else (rank + 1) % world
        prv = dist.get_global_rank(group, (rank - 1) % world) if group is not None else (rank - 1) % world
        kv_recv = [(torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
        acc_recv = [tuple(torch.empty_like(a) for a in acc) for _ in range(2)]
        cur_k, cur_v = k, v
        for t, (src, diag) in enumerate(ring_schedule(rank, world, causal)):
            kv_reqs = []
            if t + 1 < world:  # the next block's K, V travel while this one computes
                nk, nv = kv_recv[t % 2]
                kv_reqs = dist.batch_isend_irecv([
                    dist.P2POp(dist.isend, cur_k, nxt, group),
                    dist.P2POp(dist.isend, cur_v, nxt, group),
                    dist.P2POp(dist.irecv, nk, prv, group),
                    dist.P2POp(dist.irecv, nv, prv, group),
                ])
            ops.block(q, cur_k, cur_v, do, acc[0], acc[1], diag)
            # this block's accumulators move on once this rank's share is in;
            # the previous rank's (for the next block) arrive. After the last
            # step each rank holds the accumulators of its own keys.
            ndk, ndv = acc_recv[t % 2]
            acc_reqs = dist.batch_isend_irecv([
                dist.P2POp(dist.isend, acc[0], nxt, group),
                dist.P2POp(dist.isend, acc[1], nxt, group),
                dist.P2POp(dist.irecv, ndk, prv, group),
                dist.P2POp(dist.irecv, ndv, prv, group),
            ])
            for req in kv_reqs + acc_reqs:
                req.wait()
            acc, acc_recv[t % 2] = (ndk, ndv), acc
            if t + 1 < world:
                cur_k, cur_v = kv_recv[t % 2]
    ops.finish(dq)
    ops.to_bf16(acc[0], dk)
    ops.to_bf16(acc[1], dv)
    return dq, dk, dv
