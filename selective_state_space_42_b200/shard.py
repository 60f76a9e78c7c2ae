"""Splitting one selective scan over several GPUs by channel.

The chains (batch row b, channel d) of the scan are independent: each reads
its own x, Δ, z column and the B, C rows shared by every channel, and writes
its own y column and final state. A layer therefore shards over channels with
no exchange at all: rank r runs selscan_fwd on channels [d0, d1) with the
same B and C (replicated, 2·L·N elements per batch row), and the union of the
ranks' outputs is the whole layer's output. Slices are whole 128-channel
tiles where possible, so every rank keeps the TMA-staged kernel's plan.
"""
from __future__ import annotations

from typing import List, Tuple

TILE = 128  # channels per tile of the TMA-staged kernel


def channel_slices(dim: int, world: int, tile: int = TILE) -> List[Tuple[int, int]]:
    """[d0, d1) for every rank: whole tiles spread as evenly as possible (the
    first ranks take one tile more), the last slice ending at dim. Ranks past
    the number of tiles get an empty slice."""
    if world < 1 or dim < 0:
        raise ValueError("world >= 1 and dim >= 0 required")
    ntiles = -(-dim // tile)
    base, extra = divmod(ntiles, world)
    out, t = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        d0, d1 = min(t * tile, dim), min((t + n) * tile, dim)
        out.append((d0, d1))
        t += n
    return out


def channel_slice(dim: int, world: int, rank: int, tile: int = TILE) -> Tuple[int, int]:
    """This rank's [d0, d1)."""
    return channel_slices(dim, world, tile)[rank]


def shard_inputs(inp: dict, d0: int, d1: int) -> dict:
    """The inputs of one selscan_fwd call restricted to channels [d0, d1):
    x, delta, z columns and A, D, delta_bias rows sliced (made contiguous),
    B and C whole."""
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif k in ("x", "delta", "z"):
            out[k] = v[:, :, d0:d1].contiguous()
        elif k in ("A", "D", "delta_bias"):
            out[k] = v[d0:d1].contiguous()
        else:
            out[k] = v
    return out
