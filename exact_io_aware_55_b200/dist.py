"""Multi-GPU helpers.  Heads (batch x head pairs) are independent units of the
attention path, so N GPUs split them with no collective on the data path;
the only collective is the max over ranks of the measured device time."""
from __future__ import annotations


def head_range(num_heads: int, world_size: int, rank: int) -> tuple[int, int]:
    """Contiguous [start, end) slice of the flattened B*H heads owned by `rank`;
    sizes differ by at most one."""
    if world_size <= 0 or not 0 <= rank < world_size or num_heads < 0:
        raise ValueError("bad world_size / rank / num_heads")
    base, extra = divmod(num_heads, world_size)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(dist, values, device=None):
    """Element-wise max of a list of floats over all ranks (a no-op without a
    process group).  Used to time multi-GPU runs as the slowest rank."""
    if dist is None or not dist.is_available() or not dist.is_initialized():
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]
