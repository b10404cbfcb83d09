"""Host-side plumbing for running the forward pass on several GPUs.

The (batch, head) chains of the gated delta rule are independent, so the
pass shards over the batch with no collective on the data path: each rank
(one process per GPU) runs its own contiguous slice of the batch through
``gdn_fwd``.  The only collectives are the timing ones (a barrier around the
timed region and the maximum of the per-rank device times).  Everything
here is backend-agnostic (``nccl`` on GPUs, ``gloo`` in the CPU tests).
"""
from __future__ import annotations

import datetime
import os


def env_rank_world():
    """(rank, local_rank, world) from the torchrun environment; (0, 0, 1) alone."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str, timeout_s: float = 120.0, device=None):
    """Join the process group (a short timeout so ranks that wait on a dead
    peer end with an error instead of hanging)."""
    import torch.distributed as dist
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)


def batch_slice(B: int, rank: int, world: int):
    """The contiguous range of batch elements rank `rank` of `world` owns
    (sizes differ by at most one; a rank may own none)."""
    base, extra = divmod(B, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def shard(t, rank: int, world: int):
    """This rank's batch slice of a [B, ...] tensor (a view)."""
    if t is None:
        return None
    lo, hi = batch_slice(t.shape[0], rank, world)
    return t[lo:hi]


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar over all ranks (the identity alone)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()
