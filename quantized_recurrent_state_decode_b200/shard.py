"""Data-parallel partition of the decode step across processes.

Every (batch, head) tile is independent and a step exchanges nothing between
tiles, so the step shards by batch rows with no collective on the data path:
rank r owns a contiguous slice of the batch and all heads, and its outputs stay
on its GPU. The only cross-rank operation is host-side plumbing for timing
(the slowest rank's elapsed time).
"""


def batch_slice(global_batch: int, rank: int, world: int):
    """(offset, size) of rank's contiguous batch slice; sizes differ by at
    most one and the slices tile [0, global_batch) in rank order."""
    if world < 1 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("bad partition arguments")
    base, extra = divmod(global_batch, world)
    size = base + (1 if rank < extra else 0)
    offset = rank * base + min(rank, extra)
    return offset, size


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank float over the default process group (the
    value itself without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
