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


# ---------------------------------------------------------------- context parallelism over time
# The sequence is split over ranks by frames (SANA-WM summary, section 3.1, Stage 3: the
# sequence split over GPUs; cliffmar.tech article, "NVIDIA SANA-WM", training section: the
# "prefix-sum composition of GDN transition matrices").  Each rank reduces its contiguous
# frames to one affine map of the state, S_end = S_begin Phi + Psi; the maps are
# all-gathered (d_k x (d_k + d_v) fp32 per chain, ~100 KB per head); each rank composes the
# maps of the ranks before it onto the sequence's entering state and runs its own frames from
# there.  Only the state-independent stages run before the exchange; the scan, pseudo-values
# and output run after it on the same workspace.

def segment_prepare(q, k, v, alpha, beta, frame_len, workspace, *, stream=None):
    """The state-independent stages of this rank's frames (kept in `workspace`) and their map
    [B, H, d_k + d_v, d_k] (Phi rows, then Psi)."""
    import torch
    from . import binding
    B, _, H, d_k = q.shape
    d_v = v.shape[-1]
    seg_map = torch.empty((B, H, d_k + d_v, d_k), dtype=torch.float32, device=q.device)
    binding.gdn_fwd(q, k, v, alpha, beta, frame_len, None, workspace=workspace, stream=stream, phase="prepare",
                    segment_map=seg_map)
    return seg_map


def entering_state(S_in, maps, rank, *, stream=None):
    """The state entering rank `rank`'s frames: S_in (zeros if None) with the maps of ranks
    0 .. rank-1 applied in order.  maps: [world, B, H, d_k + d_v, d_k]."""
    import torch
    from . import binding
    _, B, H, rows, d_k = maps.shape
    d_v = rows - d_k
    S = (torch.zeros((B, H, d_v, d_k), dtype=torch.float32, device=maps.device) if S_in is None
         else S_in.clone().contiguous())
    if rank > 0:
        binding.apply_maps(S, maps[:rank].contiguous(), stream=stream)
    return S


def segment_finish(q, k, v, alpha, beta, frame_len, S_enter, workspace, *, o=None, stream=None):
    """Scan, pseudo-values and output of this rank's frames from the state entering them,
    on the workspace segment_prepare filled.  Returns (o, S_end)."""
    from . import binding
    return binding.gdn_fwd(q, k, v, alpha, beta, frame_len, S_enter, o=o, return_state=True,
                           workspace=workspace, stream=stream, phase="finish")


def context_parallel_forward(q, k, v, alpha, beta, frame_len, S_in=None, *, workspace, group=None, stream=None):
    """One rank's part of a forward pass whose frames are split over the ranks of `group`
    (rank r holds the r-th contiguous range of frames, in order).  One all-gather of the
    segment maps (NCCL on GPUs); no other data-path collective.  Returns (o of this rank's
    tokens, the state after them) -- the last rank's state is the sequence's final state."""
    import torch
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    seg_map = segment_prepare(q, k, v, alpha, beta, frame_len, workspace, stream=stream)
    maps = torch.empty((world,) + tuple(seg_map.shape), dtype=seg_map.dtype, device=seg_map.device)
    dist.all_gather_into_tensor(maps, seg_map, group=group)
    S = entering_state(S_in, maps, rank, stream=stream)
    return segment_finish(q, k, v, alpha, beta, frame_len, S, workspace, stream=stream)
