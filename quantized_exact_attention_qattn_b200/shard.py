"""Head sharding of one attention problem over ranks (one GPU each).

Every (batch, head) of the method is an independent problem: the per-head
RMSNorm, the K mean and the V maxima run over one head's rows, the scales are
per head, and the softmax and P.V of a query head read only its KV head.  So a
problem splits over ranks by contiguous head ranges with no exchange at all:
each rank takes the column slice of the (interleaved) Q/K/V buffer that holds
its heads, runs the whole path on it and owns those heads of the output.  Only
gathering the output into one device's [B, N, H, D] buffer would take a
collective (one all-gather); nothing in the path needs one.

The slices are plain views (no copy): a [B, N, H, D] view restricted to heads
h0 .. h1-1 keeps the strides and moves the base by h0 head rows, which the C
ABI takes as a ``qattn_bnhd`` view as it is."""
from __future__ import annotations


def shard_heads(H: int, world: int, rank: int):
    """Contiguous head range [h0, h1) of ``rank`` when H heads are split over
    ``world`` ranks, the first H % world ranks taking one head more."""
    base, rem = divmod(H, world)
    h0 = rank * base + min(rank, rem)
    return h0, h0 + base + (1 if rank < rem else 0)


def kv_shard(Hq: int, Hkv: int, world: int, rank: int):
    """(q head range, kv head range) of ``rank``: the KV heads are split and
    every rank takes the query heads that read its KV heads (Hq / Hkv each)."""
    k0, k1 = shard_heads(Hkv, world, rank)
    g = Hq // Hkv
    return (k0 * g, k1 * g), (k0, k1)


def head_slice(x, h0: int, h1: int):
    """Heads [h0, h1) of a [B, N, H, D] array or tensor, as a view."""
    return x[:, :, h0:h1]
