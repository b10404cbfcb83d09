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
