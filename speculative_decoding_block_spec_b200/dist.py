"""Host-side helpers for running the verifier on several GPUs.

Requests are independent, so verification shards by request with no
collective on the data path: every rank verifies its own slice of the batch.
Only the timing is reduced across ranks (the slowest rank sets the step time).
"""


def shard(n, rank, world):
    """Contiguous slice of n requests owned by `rank` of `world` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value, device=None):
    """Maximum of a float over all ranks of the default process group (the value itself without one)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
