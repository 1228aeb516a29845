"""Head sharding of one prefill layer over ranks (one process per GPU, no exchange step).

Every step of the path is independent per (batch row, query head): the round-robin estimate
scores a head's sampled queries against its own KV head's stride-summed keys, Top-tau selects
per (head, block row), and the block-sparse attention of a head reads only its KV head
(RRAttention, "Method": per-head round-robin sampling; GQA as in the "Experiments" models). A
layer therefore splits over W ranks by contiguous KV-head groups: rank r takes KV heads
[r Hkv/W, (r+1) Hkv/W) and the g = Hq/Hkv query heads of each of them. Nothing crosses ranks on
the data path; a caller that wants every head of O on one GPU gathers them afterwards.

The one coupling between heads is the round-robin offset o_h = (h + shift) mod S, taken on the
GLOBAL head index h. A shard whose first query head is h0 runs with shift' = (shift + h0) mod S,
so its local head i samples exactly the offset global head h0 + i would.

Host-side arithmetic only (index ranges and parameters); every shard runs the same kernels as a
whole layer.
"""
from __future__ import annotations

import dataclasses

__all__ = ["HeadShard", "head_shard", "shard_params", "take_heads"]


@dataclasses.dataclass(frozen=True)
class HeadShard:
    rank: int
    world: int
    q0: int          # first global query head of the shard
    q1: int          # one past the last
    kv0: int         # first global KV head
    kv1: int
    shift: int       # round-robin shift the shard runs with, in [0, stride)

    @property
    def heads_q(self) -> int:
        return self.q1 - self.q0

    @property
    def heads_kv(self) -> int:
        return self.kv1 - self.kv0


def head_shard(heads_q: int, heads_kv: int, stride: int, shift: int, rank: int,
               world: int) -> HeadShard:
    """The heads rank ``rank`` of ``world`` owns. Raises ValueError unless Hkv divides by the
    world size (whole GQA groups per rank) and Hq by Hkv."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if heads_kv < 1 or heads_q % heads_kv:
        raise ValueError(f"heads_q {heads_q} is not a multiple of heads_kv {heads_kv}")
    if heads_kv % world:
        raise ValueError(f"heads_kv {heads_kv} does not split over {world} ranks")
    if stride < 1:
        raise ValueError(f"stride {stride} < 1")
    g = heads_q // heads_kv
    kv_per = heads_kv // world
    kv0 = rank * kv_per
    q0 = kv0 * g
    return HeadShard(rank, world, q0, q0 + kv_per * g, kv0, kv0 + kv_per,
                     (shift + q0) % stride)


def shard_params(p, rank: int, world: int):
    """(params of the shard, HeadShard) for an ``rra_params``-like object ``p`` (the binding's
    ``RraParams``): same batch, length, head dim, block, stride, tau and scale; the shard's head
    counts and shift."""
    s = head_shard(p.heads_q, p.heads_kv, p.stride, p.shift, rank, world)
    q = type(p)(p.batch, s.heads_q, s.heads_kv, p.seqlen, p.head_dim, p.block, p.stride, s.shift,
                p.tau, p.softmax_scale)
    return q, s


def take_heads(x, lo: int, hi: int):
    """Heads [lo, hi) of a [batch, heads, ...] array or tensor, contiguous (a view when batch
    is 1, a copy otherwise)."""
    y = x[:, lo:hi]
    if hasattr(y, "contiguous"):
        return y.contiguous()
    import numpy as np
    return np.ascontiguousarray(y)
