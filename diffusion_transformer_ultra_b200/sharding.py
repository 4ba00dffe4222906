"""Head partition of one attention layer across ranks (one process per GPU).

The attention of one head reads only that head's Q, K and V, so a layer's heads split across
GPUs with no exchange between them: rank r runs heads [h0, h1) with its own plan for
h1 - h0 heads (the plan depends on the geometry, not on which heads it serves), and the ranks'
outputs, put side by side along the head axis, are the layer's output.  Inputs are the head
slices a column-parallel QKV projection leaves on each rank; this module holds no step of the
attention itself.
"""
from __future__ import annotations


def head_range(heads: int, world: int, rank: int) -> tuple[int, int]:
    """Heads [h0, h1) of `rank` out of `world`: contiguous blocks, the first heads % world
    ranks one head larger, so every head belongs to exactly one rank."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    if heads < world:
        raise ValueError(f"{heads} heads cannot be split over {world} ranks")
    base, extra = divmod(heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def head_slice(x, h0: int, h1: int):
    """Contiguous copy of heads [h0, h1) of a raster tensor [B, N_raster, heads, D]."""
    return x[:, :, h0:h1, :].contiguous()
