"""Partition of one attention layer's (stream, head) grid over ranks: streams first, then heads.

UnStep's layer (paper abstract: per-stream KV caches that keep a limited temporal window;
Table 3: each video is its own stream of causal chunks) never mixes streams or heads: the RoPE
rotates each (stream, token, head) row on its own, the ring append writes each (stream, head)
cache on its own, and the windowed attention of a (stream, head) reads only that pair's keys.
So a layer splits over GPUs with no exchange at all: each rank owns a rectangle of streams x
heads, keeps its own KV-cache shard (``LayerCache(..., shard=...)``) and reads and writes only
its rows of the activations.  Whole streams go to ranks first (a stream's cache then lives on
one GPU); only when there are more ranks than streams is a stream's head set split.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple


@dataclass(frozen=True)
class Shard:
    """Streams ``b0 .. b0+nb-1`` and heads ``h0 .. h0+nh-1`` of a layer with B streams and H heads."""
    b0: int
    nb: int
    h0: int
    nh: int

    def cells(self) -> List[Tuple[int, int]]:
        return [(b, h) for b in range(self.b0, self.b0 + self.nb)
                for h in range(self.h0, self.h0 + self.nh)]


def split(n: int, k: int) -> List[Tuple[int, int]]:
    """``n`` items in ``k`` contiguous near-equal parts (the first ``n mod k`` one larger), as
    (start, count)."""
    if k < 1 or n < k:
        raise ValueError(f"cannot split {n} items into {k} non-empty parts")
    base, extra = divmod(n, k)
    out, start = [], 0
    for i in range(k):
        cnt = base + (1 if i < extra else 0)
        out.append((start, cnt))
        start += cnt
    return out


def plan(B: int, H: int, world: int) -> List[Shard]:
    """The shard of every rank, rank order.

    ``world <= B``: each rank takes a contiguous block of whole streams with all heads.
    ``world > B``: the ranks are spread over the streams as evenly as possible (each stream gets
    ``world // B`` or one more) and each stream's heads are split among its ranks.  More ranks
    than (stream, head) pairs is an error (a rank would have nothing to do)."""
    if B < 1 or H < 1 or world < 1:
        raise ValueError("B, H and world must be positive")
    if world > B * H:
        raise ValueError(f"{world} ranks for {B * H} (stream, head) pairs")
    if world <= B:
        return [Shard(b0, nb, 0, H) for b0, nb in split(B, world)]
    shards = []
    for b, (_, ranks) in enumerate(split(world, B)):
        if ranks > H:
            raise ValueError(f"stream {b} would get {ranks} ranks for {H} heads")
        shards.extend(Shard(b, 1, h0, nh) for h0, nh in split(H, ranks))
    return shards
