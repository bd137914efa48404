"""Head-parallel sharding of one attention problem over ranks (one GPU per rank).

KV groups are independent in block-causal GQA attention: the query heads of group
g only ever read K/V head g.  Splitting the KV groups (and their query heads)
evenly over ranks therefore needs no data exchange at all, in the forward or the
backward (the head-parallel layout that Ulysses sequence parallelism converts to,
MAGI-1 research notes (zhao9797.github.io), "Inference infra > Ulysses").
"""
from __future__ import annotations


def shard_heads(hq: int, hkv: int, rank: int, world: int):
    """(q_head_begin, q_head_end, kv_head_begin, kv_head_end) owned by ``rank``."""
    if world <= 0 or not (0 <= rank < world):
        raise ValueError("bad rank/world")
    if hkv % world != 0:
        raise ValueError(f"{hkv} KV heads cannot be split evenly over {world} ranks")
    G = hq // hkv
    per = hkv // world
    g0, g1 = rank * per, (rank + 1) * per
    return g0 * G, g1 * G, g0, g1
