"""Context parallelism over time on one GPU: the sequence split into segments, each
reduced to its map S_end = S_begin Phi + Psi by the state-independent stages, the maps
composed onto the entering state, each segment finished from its own entering state.
The ranks run one after another here (one GPU); the gathered result must equal the
fp64 token loop over the whole sequence at the contract's tolerance, and a single
segment's prepare + finish must equal the one-call pass bit for bit.
(SANA-WM summary, section 3.1, Stage 3; cliffmar.tech article, "NVIDIA SANA-WM",
training section: prefix-sum composition of the GDN transition matrices.)
"""
import numpy as np
import pytest
import torch

import gated_deltanet_linear_chunkwise_b200 as g
import oracle
from gated_deltanet_linear_chunkwise_b200 import dist as gdist
from gated_deltanet_linear_chunkwise_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}


def rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.abs(x - ref).max() / np.abs(ref).max())


CASES = [
    # dtype, B, H, frames, L, d, segment boundaries (in frames)
    ("bf16", 1, 2, 6, 128, 64, (0, 2, 6)),
    ("bf16", 1, 2, 3, 880, 112, (0, 1, 2, 3)),
    ("f32", 2, 2, 5, 64, 32, (0, 3, 5)),
    ("bf16", 1, 3, 4, 100, 48, (0, 0, 4)),  # an empty segment maps every state to itself
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s_B%dH%dF%dL%d_d%d_%s" % (c[:6] + ("-".join(map(str, c[6])),)))
@pytest.mark.parametrize("regime", ["slow", "lit"])
def test_segments_compose_to_one_pass(case, regime):
    dtype, B, H, F, L, d, cuts = case
    inp = W.draw(B, H, F * L, d, d, frame_len=L, seed=51, regime=regime, dtype=dtype, state_std=0.1)
    dev = {k: (None if t is None else t.cuda().contiguous()) for k, t in inp.items()}
    segs = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        seg = {k: dev[k][:, a * L:b * L].contiguous() for k in ("q", "k", "v", "alpha", "beta")}
        T = (b - a) * L
        nbytes = max(g.workspace_bytes(B, H, T, L, d, d, dtype), 256)
        seg["ws"] = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        segs.append(seg)
    # every rank: its state-independent stages and its map
    maps = torch.stack([gdist.segment_prepare(s["q"], s["k"], s["v"], s["alpha"], s["beta"], L, s["ws"])
                        for s in segs])
    # every rank: its entering state from the maps before it, then its frames
    outs, S_end = [], None
    for r, s in enumerate(segs):
        S_enter = gdist.entering_state(dev["S_in"], maps, r)
        o_r, S_end = gdist.segment_finish(s["q"], s["k"], s["v"], s["alpha"], s["beta"], L, S_enter, s["ws"])
        outs.append(o_r)
    torch.cuda.synchronize()
    o = torch.cat(outs, dim=1).double().cpu().numpy()
    o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"])
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S_end.double().cpu(), S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_segment_map_is_the_affine_map_of_the_segment(dtype):
    # S_end = S_begin Phi + Psi for an arbitrary entering state, against the token loop
    B, H, F, L, d = 1, 2, 3, 96, 64
    inp = W.draw(B, H, F * L, d, d, frame_len=L, seed=53, regime="slow", dtype=dtype, state_std=0.3)
    dev = {k: (None if t is None else t.cuda().contiguous()) for k, t in inp.items()}
    ws = torch.empty(g.workspace_bytes(B, H, F * L, L, d, d, dtype), dtype=torch.uint8, device="cuda")
    m = gdist.segment_prepare(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], L, ws)
    torch.cuda.synchronize()
    m = m.double().cpu().numpy()
    Phi, Psi = m[:, :, :d], m[:, :, d:]
    S0 = inp["S_in"].double().numpy()
    _, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], inp["S_in"])
    assert rel(np.einsum("bhvk,bhkl->bhvl", S0, Phi) + Psi, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prepare_then_finish_equals_one_call(dtype):
    B, H, F, L, d = 1, 2, 3, 128, 64
    inp = W.draw(B, H, F * L, d, d, frame_len=L, seed=55, regime="slow", dtype=dtype, state_std=0.1)
    dev = {k: (None if t is None else t.cuda().contiguous()) for k, t in inp.items()}
    ws = torch.empty(g.workspace_bytes(B, H, F * L, L, d, d, dtype), dtype=torch.uint8, device="cuda")
    o1, S1 = g.gdn_fwd(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], L, dev["S_in"], return_state=True,
                       workspace=ws)
    g.gdn_fwd(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], L, None, workspace=ws, phase="prepare")
    o2, S2 = g.gdn_fwd(dev["q"], dev["k"], dev["v"], dev["alpha"], dev["beta"], L, dev["S_in"], return_state=True,
                       workspace=ws, phase="finish")
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
