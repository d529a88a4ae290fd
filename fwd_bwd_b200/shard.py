"""Data-parallel partition of SageBwd attention across ranks.

Every (batch, head) pair is an independent problem -- the prologue's K mean, every block
scale, the forward and the backward are all per head, and the operator has no weights -- so a
global batch is split into contiguous ranges of flattened heads ``bh = b * H + h`` with no
exchange on the data path.  The ranges differ in size by at most one head.
"""
from __future__ import annotations


def head_range(total_heads: int, world: int, rank: int) -> range:
    """Contiguous slice of ``range(total_heads)`` owned by ``rank`` of ``world``."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(total_heads, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))
