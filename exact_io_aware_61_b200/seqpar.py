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
