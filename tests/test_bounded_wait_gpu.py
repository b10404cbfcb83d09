"""A bounded device-side wait that gives up (no GPU fault, trap or hang).

The debug switch GDN_DEBUG_DROP_SIGNAL=1 makes the diagonal-inverse kernel
withhold its first block's Gram product, so the wait on it can never complete;
GDN_DEBUG_WAIT_LIMIT_US shortens the waits' limit from 2 s to 1 ms.  The
waiting thread records a timeout in the pass's error word, the block's other
threads skip their work, TMEM is released, and the later kernels of the pass
skip theirs.  The host then
learns it through the status word (asynchronous calls) or GDN_ERR_TIMEOUT
(synchronous calls), and the next call on the same context is correct.
"""
import ctypes

import numpy as np
import pytest
import torch

import gated_deltanet_linear_chunkwise_b200 as g
import oracle
from gated_deltanet_linear_chunkwise_b200 import workloads as W
from gated_deltanet_linear_chunkwise_b200.binding import NUM_STAGES, GdnError

pytestmark = pytest.mark.gpu

GDN_ERR_TIMEOUT = 7


def rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / np.abs(ref).max())


def test_wait_gives_up_then_context_is_usable(monkeypatch):
    L = 128
    inp = W.draw(1, 2, 3 * L, 64, 64, frame_len=L, seed=41, regime="slow", dtype="bf16", state_std=0.1)
    d = {k: (None if v is None else v.cuda().contiguous()) for k, v in inp.items()}

    def call(**kw):
        return g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], L, d["S_in"], return_state=True, **kw)

    monkeypatch.setenv("GDN_DEBUG_WAIT_LIMIT_US", "1000")
    monkeypatch.setenv("GDN_DEBUG_DROP_SIGNAL", "1")
    # asynchronous call: it returns at once; the status word, written in stream order, says the
    # pass gave up
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    call(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) != 0
    # a synchronous call (stage timing) reports the same as a status code
    with pytest.raises(GdnError) as ei:
        call(stage_ms=(ctypes.c_float * NUM_STAGES)())
    assert ei.value.status == GDN_ERR_TIMEOUT
    monkeypatch.delenv("GDN_DEBUG_DROP_SIGNAL")
    monkeypatch.delenv("GDN_DEBUG_WAIT_LIMIT_US")

    # the context is intact: the same call now completes, reports 0 and matches the oracle
    st.fill_(5)
    o, S = call(status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"])
    assert rel(o.double().cpu(), o_ref) <= 2e-2
    assert rel(S.double().cpu(), S_ref) <= 2e-2
