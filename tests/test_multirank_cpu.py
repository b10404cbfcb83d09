"""The multi-rank path on the CPU: two gloo ranks shard a batch the way
``bench.py --gpus N`` does, each runs its slice through the fp64 oracle, and
the gathered result equals the unsharded pass; the timing reduction takes
the maximum over ranks.  No GPU is involved."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from gated_deltanet_linear_chunkwise_b200 import dist as gdist
from gated_deltanet_linear_chunkwise_b200 import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    gdist.init("gloo", timeout_s=60)
    try:
        assert gdist.env_rank_world() == (rank, rank, world)
        # every rank draws the same full batch from the shared seed and keeps its slice
        inp = W.draw(3, 2, 2 * 16, 8, 8, frame_len=16, seed=11, regime="slow", dtype="f32", state_std=0.1)
        mine = {k: gdist.shard(v, rank, world) for k, v in inp.items()}
        o, S = oracle.token_recurrence(mine["q"], mine["k"], mine["v"], mine["alpha"], mine["beta"],
                                       mine["S_in"], nthreads=1)
        # gather the per-rank outputs (ragged: 2 + 1 batch elements)
        shapes = [None] * world
        dist.all_gather_object(shapes, (o.tolist(), S.tolist()))
        # timing reduction: the maximum of per-rank values
        t = gdist.max_over_ranks(10.0 + rank)
        gdist.barrier()
        if rank == 0:
            results.put((shapes, t))
    finally:
        dist.destroy_process_group()


def test_batch_slices_cover_the_batch():
    for B in (0, 1, 2, 3, 7, 8):
        for world in (1, 2, 3, 8):
            got = [gdist.batch_slice(B, r, world) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [hi - lo for lo, hi in got]
            assert max(sizes) - min(sizes) <= 1


def test_max_over_ranks_alone_is_identity():
    assert gdist.max_over_ranks(3.5) == 3.5


@pytest.mark.timeout(240)
def test_two_gloo_ranks_shard_equals_unsharded():
    import oracle
    world = 2
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=200)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    parts, t = results.get(timeout=5)
    assert t == 11.0
    o = np.concatenate([np.asarray(p[0]) for p in parts if len(p[0])], axis=0)
    S = np.concatenate([np.asarray(p[1]) for p in parts if len(p[1])], axis=0)
    inp = W.draw(3, 2, 2 * 16, 8, 8, frame_len=16, seed=11, regime="slow", dtype="f32", state_std=0.1)
    o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"],
                                           nthreads=1)
    assert np.array_equal(o, o_ref) and np.array_equal(S, S_ref)


# ---------------------------------------------------------------- context parallelism over time
# The protocol of the context-parallel split (frames over ranks): each rank reduces its
# contiguous range of frames to one affine map of the state, S_out = S_in Phi_r + C_r, the
# maps are all-gathered, each rank composes the maps of the ranks before it onto S_in to get
# its entering state, and runs its own frames from there.  Here the oracle stands in for the
# kernels; the test pins the orientation of the maps, the order of the composition and the
# frame ranges.

def _segment_map(seg, d_k):
    """(Phi, C) of a segment: C = the final state from a zero state; row j of Phi = the
    final state from S_in = e_j in row 0, minus C (the map is affine in S_in)."""
    import oracle
    B, T, H, _ = seg["q"].shape
    d_v = seg["v"].shape[-1]
    _, C = oracle.token_recurrence(seg["q"], seg["k"], seg["v"], seg["alpha"], seg["beta"], None, nthreads=1)
    Phi = np.zeros((B, H, d_k, d_k))
    for j in range(d_k):
        E = np.zeros((B, H, d_v, d_k))
        E[:, :, 0, j] = 1.0
        _, Sj = oracle.token_recurrence(seg["q"], seg["k"], seg["v"], seg["alpha"], seg["beta"], E, nthreads=1)
        Phi[:, :, j, :] = Sj[:, :, 0, :] - C[:, :, 0, :]
    return Phi, C


def _cp_worker(rank, world, port, results):
    import torch.distributed as dist
    import oracle
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    gdist.init("gloo", timeout_s=60)
    try:
        F, L, d_k, d_v = 7, 12, 6, 5
        inp = W.draw(1, 2, F * L, d_k, d_v, frame_len=L, seed=13, regime="slow", dtype="f32", state_std=0.3)
        x = {k: inp[k].double().numpy() for k in ("q", "k", "v", "alpha", "beta")}
        f0, f1 = gdist.batch_slice(F, rank, world)  # this rank's frames
        seg = {k: v[:, f0 * L:f1 * L] for k, v in x.items()}
        Phi, C = _segment_map(seg, d_k)
        maps = [None] * world
        dist.all_gather_object(maps, (Phi.tolist(), C.tolist()))
        S = inp["S_in"].double().numpy()
        for j in range(rank):  # exclusive prefix: the ranks before this one, in order
            S = np.einsum("bhvk,bhkl->bhvl", S, np.asarray(maps[j][0])) + np.asarray(maps[j][1])
        o, S_out = oracle.token_recurrence(seg["q"], seg["k"], seg["v"], seg["alpha"], seg["beta"], S,
                                           nthreads=1)
        parts = [None] * world
        dist.all_gather_object(parts, (o.tolist(), S_out.tolist()))
        gdist.barrier()
        if rank == 0:
            results.put(parts)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_protocol_on_gloo_ranks(world):
    import oracle
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_cp_worker, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=200)
    for p in procs:
        if p.is_alive():
            p.kill()
        assert p.exitcode == 0
    parts = results.get(timeout=5)
    F, L, d_k, d_v = 7, 12, 6, 5
    inp = W.draw(1, 2, F * L, d_k, d_v, frame_len=L, seed=13, regime="slow", dtype="f32", state_std=0.3)
    o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"],
                                           nthreads=1)
    o = np.concatenate([np.asarray(p[0]) for p in parts if np.asarray(p[0]).size], axis=1)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12 * np.abs(o_ref).max())
    np.testing.assert_allclose(np.asarray(parts[-1][1]), S_ref, rtol=0, atol=1e-12 * np.abs(S_ref).max())
