"""Splitting one attention problem over several GPUs by (batch entry, KV head).

A query head reads only its own KV head, and every KV head's group of g query
heads is independent of the others (GQA summary, "The idea": one key and one
value head per group), so the B * H_kv (batch entry, KV head) units of a
problem can be computed on different GPUs with no exchange, forward or
backward: dK and dV of a KV head are reduced over its group on the GPU that
holds the group.  Each rank takes a contiguous run of units in (b, kvh) order.
A run is computed as one call when it is a rectangle: whole batch entries with
all their heads, or a range of KV heads of one batch entry (with their query
heads); shard_block returns that rectangle.

The tensors stay [B, N, H, dh]: a rank's inputs are the slices
q[b0:b1, :, g*k0:g*k1], k[b0:b1, :, k0:k1], v[b0:b1, :, k0:k1] made contiguous,
and its outputs are the same slices of out, lse, dq, dk and dv.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Block:
    b0: int  # batch entries [b0, b1)
    b1: int
    k0: int  # KV heads [k0, k1); query heads [g k0, g k1)
    k1: int


def shard_block(B: int, H_kv: int, world: int, rank: int) -> Block:
    """This rank's rectangle of (batch entry, KV head) units.  The B * H_kv
    units must split evenly into rectangles: world divides B (whole batch
    entries per rank), or B * H_kv / world divides H_kv (KV-head ranges within
    a batch entry).  Raises ValueError otherwise."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank must be in [0, world)")
    n = B * H_kv
    if n % world:
        raise ValueError(f"{n} (batch entry, KV head) units do not split over {world} ranks")
    per = n // world
    lo = rank * per
    if per % H_kv == 0:  # whole batch entries
        b0 = lo // H_kv
        return Block(b0, b0 + per // H_kv, 0, H_kv)
    if H_kv % per == 0:  # a range of KV heads of one batch entry
        b, k0 = divmod(lo, H_kv)
        return Block(b, b + 1, k0, k0 + per)
    raise ValueError(f"{per} units per rank are neither whole batch entries nor a divisor of H_kv={H_kv}")


def q_heads(blk: Block, g: int) -> slice:
    return slice(g * blk.k0, g * blk.k1)


def kv_heads(blk: Block) -> slice:
    return slice(blk.k0, blk.k1)


def take(t, blk: Block, heads: slice):
    """The block of a [B, N, H, dh] tensor, contiguous (a copy when the block
    does not hold every head)."""
    return t[blk.b0:blk.b1, :, heads].contiguous()


def take_lse(lse, blk: Block, g: int):
    """The block of an lse tensor [B, H_q, N]."""
    return lse[blk.b0:blk.b1, q_heads(blk, g)].contiguous()
