"""Splitting the fused Q/K RMSNorm + RoPE work across ranks.

Every token is independent: its norm spans only its own row and its angles
depend only on its position. A sequence (or a batch of sequences) therefore
splits into contiguous token ranges, one per rank, with no exchange. A 3D
shard passes pos_offset so that its first token takes the patch position it
has in the whole sequence; a table-form shard takes the matching rows of the
cos/sin table.
"""
from __future__ import annotations

from typing import Tuple


def token_shard(num_tokens: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced [start, start + count) of `num_tokens` for `rank`
    of `world` (the first num_tokens % world ranks take one token more)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside world of {world}")
    if num_tokens < 0:
        raise ValueError("num_tokens < 0")
    base, extra = divmod(num_tokens, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def shard_pos_offset(start: int, pos_offset: int, patches: int) -> int:
    """pos_offset of a 3D shard that starts `start` tokens into a call whose
    own pos_offset is `pos_offset`, on a ppf*pph*ppw = `patches` grid."""
    if patches < 1:
        raise ValueError("patches < 1")
    return (pos_offset + start) % patches
