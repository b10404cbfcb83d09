"""gdn_fwd_noalloc: the forward pass for callers that cannot allocate device
memory (its scratch is a fixed device array inside the library).  It must
give what gdn_fwd gives, call after call, through the C ABI.

This file is collected last on purpose, so a run that stops at its first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import gated_deltanet_linear_chunkwise_b200 as g
import oracle
from gated_deltanet_linear_chunkwise_b200 import workloads as W

TOL = 2e-2  # the bf16-input bar the parity tests use
FAKE = 1 << 40  # never dereferenced: these calls are rejected before any launch


def _lib():
    lib = g.load_library()
    fn = lib.gdn_fwd_noalloc
    V, I, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    fn.argtypes = [V, V, V, V, V, V, V, V, I, I, LL, I, I, I, V]
    fn.restype = I
    return lib


def test_noalloc_rejects_oversized_and_invalid():
    lib = _lib()
    # 8 x 20 frame-heads of 880 tokens need ~213 MB of scratch: more than the fixed array
    rc = lib.gdn_fwd_noalloc(FAKE, FAKE + 2 ** 30, FAKE + 2 ** 31, FAKE + 2 ** 32, FAKE + 2 ** 33, None, None,
                             FAKE + 2 ** 34, 8, 20, 880, 880, 112, 112, None)
    assert rc == 3  # GDN_ERR_UNSUPPORTED
    assert "scratch" in g.last_error()
    rc = lib.gdn_fwd_noalloc(FAKE, FAKE + 2 ** 30, FAKE + 2 ** 31, FAKE + 2 ** 32, FAKE + 2 ** 33, None, None,
                             FAKE + 2 ** 34, 1, 2, 100, 64, 64, 64, None)
    assert rc == 2  # GDN_ERR_SHAPE: T not a multiple of frame_len


def _rel(x, ref):
    x = x.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.mark.gpu
def test_noalloc_matches_gdn_fwd_twice():
    import torch

    lib = _lib()
    L, d, B, H = 880, 112, 2, 4
    stream = torch.cuda.current_stream()
    # leave an error text behind on this thread; a successful call must clear it
    assert lib.gdn_fwd_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 1, 2, 100, 64, 64, 64, None) == 2
    assert g.last_error() != ""
    for call, (seed, with_state) in enumerate([(11, True), (12, False)]):
        inp = W.draw(B, H, 2 * L, d, d, frame_len=L, seed=seed, regime="slow", dtype="bf16", state_std=0.05)
        dv = {k: (None if t is None else t.cuda().contiguous()) for k, t in inp.items()}
        S_in = dv["S_in"] if with_state else None
        # the existing entry point
        o_ref, S_ref = g.gdn_fwd(dv["q"], dv["k"], dv["v"], dv["alpha"], dv["beta"], L, S_in,
                                 return_state=True)
        # the no-allocation entry point, through the C ABI
        o = torch.full_like(o_ref, float("nan"))
        S = torch.full_like(S_ref, float("nan"))
        rc = lib.gdn_fwd_noalloc(dv["q"].data_ptr(), dv["k"].data_ptr(), dv["v"].data_ptr(),
                                 dv["alpha"].data_ptr(), dv["beta"].data_ptr(),
                                 None if S_in is None else S_in.data_ptr(), S.data_ptr(), o.data_ptr(),
                                 B, H, 2 * L, L, d, d, stream.cuda_stream)
        assert rc == 0, g.last_error()
        assert g.last_error() == ""  # no stale text from an earlier failure
        torch.cuda.synchronize()
        assert torch.isfinite(o.float()).all() and torch.isfinite(S).all()
        assert _rel(o, o_ref) <= TOL, ("call", call)
        assert _rel(S, S_ref) <= TOL, ("call", call)
        # and against the fp64 token loop itself, at the same bar
        S0 = None if S_in is None else inp["S_in"]
        o_ora, S_ora = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], S0)
        assert _rel(o, torch.from_numpy(o_ora)) <= TOL, ("call", call)
        assert _rel(S, torch.from_numpy(S_ora)) <= TOL, ("call", call)
