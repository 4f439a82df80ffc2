"""Request sharding across ranks (one process per GPU).

Requests are independent: the rule reads only a request's own rows, and its
random numbers are keyed by the request's GLOBAL index.  A batch of B requests
therefore splits into contiguous slices, one per rank, each verified with
request_offset = the slice's first global index, and the concatenated outputs
equal those of one call over the whole batch.  There is no exchange on the data
path; the only collective is the timing reduction (max over ranks).
"""


def shard_range(B: int, world: int, rank: int):
    """[start, stop) of rank's contiguous slice of B requests (sizes differ by <= 1)."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    stop = start + base + (1 if rank < extra else 0)
    return start, stop


def max_over_ranks(value: float, device=None) -> float:
    """The largest `value` over all ranks of the default process group (the
    step time every rank waits for); the value itself without one."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
