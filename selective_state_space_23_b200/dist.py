"""Multi-process (one process per GPU) plumbing for the scan.

The selective scan is independent across batch rows and channels (each channel's recurrence
only reads its own inputs and the per-row B_t, C_t), so a batch is sharded across ranks with no
data exchange: each rank scans its rows and nothing is communicated on the forward data path.
The backward of a batch-sharded step has one exchange: the per-channel parameter gradients
(dA [dim, N], dD and ddt_bias [dim]) are sums over every (row, step) and so over the ranks'
rows; :func:`allreduce_param_grads` sums them with one all-reduce.  Every other gradient (du,
dδ, dz, dB, dC, dh0) belongs to the rank's own rows.  The remaining collectives are host-side
timing plumbing: a barrier and the maximum of per-rank times.
"""
from typing import Dict, Sequence, Tuple

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


PARAM_GRADS = ("dA", "dD", "ddt_bias")


def allreduce_param_grads(grads: Dict[str, torch.Tensor],
                          keys: Sequence[str] = PARAM_GRADS) -> Dict[str, torch.Tensor]:
    """Sum ``grads[k]`` for ``k`` in ``keys`` over the ranks of the default process group, in
    place, as one all-reduce of a single flat bucket (the tensors share one dtype and device:
    fp32 on the GPU for the library's gradients).  Keys that are absent or None are skipped; every
    rank must pass the same keys and shapes, since all ranks take the same collective.  Without an
    initialised group of more than one rank, ``grads`` is returned unchanged."""
    import torch.distributed as dist
    present = [k for k in keys if grads.get(k) is not None]
    if not present or not (dist.is_available() and dist.is_initialized()) \
            or dist.get_world_size() == 1:
        return grads
    flat = torch.cat([grads[k].reshape(-1) for k in present])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM)
    off = 0
    for k in present:
        n = grads[k].numel()
        grads[k].copy_(flat[off:off + n].view_as(grads[k]))
        off += n
    return grads
