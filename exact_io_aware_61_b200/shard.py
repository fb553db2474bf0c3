"""Partition of the attention work across GPUs by (batch, KV head) pairs.

Each (batch, KV head) pair is an independent problem: the forward's query
heads read only their own KV head's K and V, and the backward's dK and dV of a
KV head sum only over that head's group of query heads (fanfani.net
"FlashAttention", "Do not materialize the matrix": every head's tile stream
touches its own Q, K and V and nothing else). So a job over ``B * Hkv`` pairs
splits into contiguous ranges of pairs, one per rank, with no exchange on the
data path.

In the dense ``[B][H][N][d]`` layout the flattened head index is
``b * H + h``. A contiguous range of pairs ``[p0, p1)`` is then a contiguous
range of flattened KV heads (K, V, dK, dV), and, because a KV head's query
heads are adjacent (query head ``h`` reads KV head ``h // g``), the contiguous
range ``[p0 * g, p1 * g)`` of flattened query heads (Q, O, dO, dQ, LSE). Each
rank therefore runs the library on plain views of its slice with ``B = 1``,
``Hq = (p1 - p0) * g`` and ``Hkv = p1 - p0``, and the head mapping inside the
slice is the same contiguous grouping.
"""

from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class PairShard:
    """Rank ``rank``'s share ``[p0, p1)`` of the ``B * Hkv`` (batch, KV head) pairs."""

    B: int
    Hq: int
    Hkv: int
    p0: int
    p1: int

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    @property
    def pairs(self) -> int:
        return self.p1 - self.p0

    @property
    def q_heads(self) -> tuple:
        """Flattened query-head range ``[h0, h1)`` of the shard."""
        return self.p0 * self.group, self.p1 * self.group

    @property
    def kv_heads(self) -> tuple:
        """Flattened KV-head range ``[h0, h1)`` of the shard."""
        return self.p0, self.p1

    def local_shape(self) -> tuple:
        """``(B, Hq, Hkv)`` of the shard's problem as the library sees it:
        whole batch entries when the shard starts and ends on a batch
        boundary, else one batch entry of ``pairs`` KV heads."""
        if self.p0 % self.Hkv == 0 and self.p1 % self.Hkv == 0:
            return self.pairs // self.Hkv, self.Hq, self.Hkv
        return 1, self.pairs * self.group, self.pairs


def pair_range(B: int, Hq: int, Hkv: int, rank: int, world: int) -> PairShard:
    """Balanced contiguous split of the ``B * Hkv`` pairs over ``world`` ranks.

    The first ``(B * Hkv) % world`` ranks take one pair more than the others;
    a rank may receive no pair when there are fewer pairs than ranks.
    """
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if Hq < 1 or Hkv < 1 or Hq % Hkv != 0 or B < 0:
        raise ValueError("need B >= 0 and Hq a positive multiple of Hkv")
    P = B * Hkv
    base, rem = divmod(P, world)
    p0 = rank * base + min(rank, rem)
    p1 = p0 + base + (1 if rank < rem else 0)
    return PairShard(B, Hq, Hkv, p0, p1)


def q_view(t, shard: PairShard):
    """The shard's slice of a query-side tensor ``[B, Hq, N, ...]`` in its local shape."""
    h0, h1 = shard.q_heads
    bl, hql, _ = shard.local_shape()
    flat = t.reshape(t.shape[0] * t.shape[1], *t.shape[2:])
    return flat[h0:h1].reshape(bl, hql, *t.shape[2:])


def kv_view(t, shard: PairShard):
    """The shard's slice of a KV-side tensor ``[B, Hkv, N, d]`` in its local shape."""
    h0, h1 = shard.kv_heads
    bl, _, hkvl = shard.local_shape()
    flat = t.reshape(t.shape[0] * t.shape[1], *t.shape[2:])
    return flat[h0:h1].reshape(bl, hkvl, *t.shape[2:])
