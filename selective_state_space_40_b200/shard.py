"""Data-parallel sharding of one selective-scan call over ranks (host logic).

The scan's channels (batch row b, channel d) are independent: the pages'
recurrence runs per channel and state with nothing shared between channels
except B and C, which are per batch row. A call therefore shards over (b, d)
with no exchange between ranks: each rank scans its own block of batch rows
or of channels, and the results are the unsharded call's, element for element.

``shard_range`` picks the block: whole batch rows when the rows split evenly
over the ranks, otherwise contiguous channel blocks of a multiple of 8
channels (so a rank's rows keep the 16-byte alignment the vector and TMA
paths want). ``shard_views`` returns the rank's views of the call's tensors:
the same strides as the full tensors, the data pointers offset by the block's
start, and the per-channel parameters (A, D, delta_bias) sliced by channel.
"""
from __future__ import annotations

from typing import Dict, Tuple


def shard_range(batch: int, dim: int, world: int, rank: int) -> Tuple[int, int, int, int]:
    """(b0, b1, d0, d1): the batch rows [b0, b1) and channels [d0, d1) of this
    rank. Every (b, d) belongs to exactly one rank; a rank may get nothing
    (b0 == b1 or d0 == d1) when there is less work than ranks."""
    if not 0 <= rank < world:
        raise ValueError("rank outside [0, world)")
    if batch % world == 0:
        per = batch // world
        return rank * per, (rank + 1) * per, 0, dim
    units = (dim + 7) // 8
    u0, u1 = units * rank // world, units * (rank + 1) // world
    return 0, batch, min(dim, 8 * u0), min(dim, 8 * u1)


_PER_CHANNEL = ("u", "delta", "z", "y")      # [b, d, L]
_PER_ROW = ("B", "C")                        # [b, N, L]
_PER_PARAM = ("A", "D", "delta_bias")        # [d, ...]
_PER_STATE = ("initial_state", "last_state")  # [b, d, N]


def shard_views(tensors: Dict[str, object], batch: int, dim: int, world: int, rank: int) -> Dict[str, object]:
    """The rank's views (no copies) of a scan call's tensors, keyed as in
    ``tensors``; None entries stay None."""
    b0, b1, d0, d1 = shard_range(batch, dim, world, rank)
    out = {}
    for k, t in tensors.items():
        if t is None:
            out[k] = None
        elif k in _PER_CHANNEL or k in _PER_STATE:
            out[k] = t[b0:b1, d0:d1]
        elif k in _PER_ROW:
            out[k] = t[b0:b1]
        elif k in _PER_PARAM:
            out[k] = t[d0:d1]
        else:
            raise KeyError(f"unknown scan argument {k}")
    return out
