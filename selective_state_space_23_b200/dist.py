"""Multi-process (one process per GPU) plumbing for the scan.

The selective scan is independent across batch rows and channels (each channel's recurrence
only reads its own inputs and the per-row B_t, C_t), so a batch is sharded across ranks with no
data exchange: each rank scans its rows and nothing is communicated on the data path.  The only
collectives are host-side timing plumbing: a barrier and the maximum of per-rank times.
"""
from typing import Tuple

import torch


def shard_rows(total_rows: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [begin, end) of batch rows owned by ``rank`` (sizes differ by at most one)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} for world size {world}")
    if total_rows < 0:
        raise ValueError("total_rows must be non-negative")
    base, extra = divmod(total_rows, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of ``value`` over all ranks of the default process group (the value itself when
    torch.distributed is not initialised)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
