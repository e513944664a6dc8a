"""Multi-process (one process per GPU) plumbing for the scan.

Three ways to shard one scan over GPUs:

* batch rows (below): independent, no exchange in the forward;
* channels (:func:`shard_channels`): independent too; the backward's dB, dC are sums over the
  channels and take one all-reduce (:func:`allreduce_bc_grads`), while dA, dD, ddt_bias belong
  to the rank's own channels;
* the sequence (:func:`seq_split_scan_fwd`): each GPU holds a segment of the time axis; one
  all-gather of the segments' (end state, ΣΔ) summaries, a local chain over the earlier
  segments, then each GPU's forward from its true entering state.

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


def shard_channels(dim: int, world: int, rank: int, align: int = 16) -> Tuple[int, int]:
    """Contiguous [begin, end) of channels d owned by ``rank``: whole blocks of ``align``
    channels (16: the kernels' warps of channels; 64: the chunked form's tiles), the ranks'
    block counts differing by at most one, the last block cut at ``dim``.  The rank scans the
    channel slice of u, delta, z (a strided view, or a copy) with the matching rows of A, D and
    dt_bias, and the whole B, C of its batch rows."""
    if align <= 0:
        raise ValueError("align must be positive")
    if dim < 0:
        raise ValueError("dim must be non-negative")
    b0, b1 = shard_rows((dim + align - 1) // align, world, rank)
    return min(dim, b0 * align), min(dim, b1 * align)


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


BC_GRADS = ("dB", "dC")


def allreduce_bc_grads(grads: Dict[str, torch.Tensor],
                       keys: Sequence[str] = BC_GRADS) -> Dict[str, torch.Tensor]:
    """Channel-sharded backward: sum ``grads["dB"]``, ``grads["dC"]`` (each rank's sums over its
    own channels) over the ranks of the default process group, in place, as one all-reduce of a
    single flat bucket.  16-bit gradients are summed in f32 and rounded once at the end; f32 and
    f64 ones in their own type.  The same rules as :func:`allreduce_param_grads` for absent keys,
    shapes and a missing or single-rank group."""
    import torch.distributed as dist
    present = [k for k in keys if grads.get(k) is not None]
    if not present or not (dist.is_available() and dist.is_initialized()) \
            or dist.get_world_size() == 1:
        return grads
    acc = grads[present[0]].dtype
    if acc in (torch.bfloat16, torch.float16):
        acc = torch.float32
    flat = torch.cat([grads[k].reshape(-1).to(acc) for k in present])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM)
    off = 0
    for k in present:
        n = grads[k].numel()
        grads[k].copy_(flat[off:off + n].view_as(grads[k]))
        off += n
    return grads


def _library_ops(scalar_a: bool, zoh: bool):
    import selective_state_space_23_b200 as ssm

    def summary(u, delta, A, B, C, dt_bias, delta_softplus):
        return ssm.ssm_scan_fwd_summary(u, delta, A, B, C, dt_bias=dt_bias,
                                        delta_softplus=delta_softplus, scalar_a=scalar_a, zoh=zoh)

    def chain(hend_all, dsum_all, A, h0):
        return ssm.ssm_scan_chain(hend_all, dsum_all, A, h0=h0, scalar_a=scalar_a)

    def scan(u, delta, A, B, C, D, z, dt_bias, delta_softplus, h0, return_final_state):
        f = ssm.ssm_scan_fwd_scalar_a if scalar_a else ssm.ssm_scan_fwd
        return f(u, delta, A, B, C, D=D, z=z, dt_bias=dt_bias, delta_softplus=delta_softplus,
                 h0=h0, return_final_state=return_final_state, zoh=zoh)

    return {"summary": summary, "chain": chain, "scan": scan}


def seq_split_scan_fwd(u, delta, A, B, C, D=None, z=None, dt_bias=None, delta_softplus=True,
                       h0=None, return_final_state=False, scalar_a=False, zoh=False, group=None,
                       ops=None):
    """Forward scan of a sequence split along time over the ranks of ``group``: rank r holds
    steps [t_r, t_{r+1}) of every time-indexed input (u, delta, z [batch, dim, L_r]; B, C
    [batch, N, L_r] or [batch, G, N, L_r]), in rank order; A, D, dt_bias and h0 (the state
    before the first step, or None) are the same on every rank.

    The scan composes affine maps of the state (the associative scan of "Temel Fikirler" on the
    Mamba summary page), so:

    1. each rank summarises its segment as h -> exp(A ΣΔ) h + hend (``summary``);
    2. one all-gather gives every rank every segment's (hend, ΣΔ), the only exchange step;
    3. each rank chains the maps of the segments before its own, starting from h0 (``chain``);
    4. each rank runs its segment's forward from that entering state (``scan``).

    Returns the rank's outputs (and its segment's final state; the last rank's is the
    sequence's).  ``ops`` replaces the three library calls (the CPU tests pass stand-ins built
    on the fp64 oracle); every rank takes the same collective.
    """
    import torch.distributed as dist
    ops = ops or _library_ops(scalar_a, zoh)
    hend, dsum = ops["summary"](u, delta, A, B, C, dt_bias, delta_softplus)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        world = dist.get_world_size(group)
        rank = dist.get_rank(group)
        packed = torch.cat([hend.reshape(-1), dsum.reshape(-1)])
        parts = [torch.empty_like(packed) for _ in range(world)]
        dist.all_gather(parts, packed, group=group)
        nh = hend.numel()
        hend_all = torch.stack([p[:nh].view_as(hend) for p in parts])
        dsum_all = torch.stack([p[nh:].view_as(dsum) for p in parts])
    else:
        rank = 0
        hend_all, dsum_all = hend.unsqueeze(0), dsum.unsqueeze(0)
    hin = ops["chain"](hend_all, dsum_all, A, h0)[rank]
    return ops["scan"](u, delta, A, B, C, D, z, dt_bias, delta_softplus, hin, return_final_state)
