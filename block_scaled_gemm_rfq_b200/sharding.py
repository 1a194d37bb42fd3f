"""Data-parallel sharding of the RFQ linear layer across ranks (one process per GPU).

The layer has no exchange step: quantization is independent per (row, 32-element
block) and the GEMM is independent per output row, so a batch of tokens splits into
contiguous row slabs, each rank quantizing and multiplying its own slab against a
replicated weight.  No collective touches the data path; the only collective here is
the scalar max used to time a step across ranks.
"""
from __future__ import annotations

TILE_ROWS = 256   # rows of one CTA-pair output tile of the GEMM


def row_slab(M: int, rank: int, world: int, align: int = TILE_ROWS):
    """[start, stop) rows of an M-row batch owned by `rank` of `world`.

    Slabs are contiguous, cover [0, M) exactly once, differ in size by at most one
    `align`-row tile, and start on a multiple of `align` (whole GEMM tiles per rank;
    the last slab takes the ragged tail)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    tiles = (M + align - 1) // align
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(t0 * align, M), min(t1 * align, M)


def max_over_ranks(value: float) -> float:
    """Max of a host scalar over the default process group (identity without one).
    Uses a CUDA tensor under NCCL and a CPU tensor under gloo."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
