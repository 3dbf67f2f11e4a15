"""Token sharding across GPUs (one process per GPU).

Tokens are independent in the ButterflyMoE forward, and the weights (packed
base, angles, router) are small enough to replicate, so a batch shards by
tokens with no collective on the data path.  The only cross-rank step is
measurement: the max over ranks of the device time.
"""
from __future__ import annotations


def token_range(total_tokens: int, rank: int, world: int):
    """Contiguous [start, end) slice of ``total_tokens`` owned by ``rank``;
    slices differ in size by at most one token and cover every token once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("need 0 <= rank < world")
    base, extra = divmod(total_tokens, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, group=None) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    backend = dist.get_backend(group)
    dev = torch.device("cuda", torch.cuda.current_device()) if backend == "nccl" else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
