"""Parity of the q/k prologue (``norm_keys`` / ``norm_queries``) through the C
ABI: the operator run on ReLU(RMSNorm(.)) features (keys further divided by
sqrt(d_k * frame_len); SANA-WM summary, "Memory-Efficient Long-Context
Modeling (Section 3.2)", paragraph "Algebraic Stabilization for Spatial
Token Explosion") against the oracle run on the oracle's own feature maps of
the same raw inputs.  Bars as elsewhere: 1e-5 fp32, 2e-2 bf16.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import gated_deltanet_linear_chunkwise_b200 as g
from gated_deltanet_linear_chunkwise_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "bf16": 2e-2}
NTHREADS = os.cpu_count() or 1


def rel(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / (den if den > 0 else 1.0))


def raw_inputs(B, H, F, L, dk, dv, dtype, seed, state_std=0.0):
    """Workload draws with q and k given per-token magnitudes (raw projections are
    not unit vectors), so the RMS normalisation has work to do."""
    inp = W.draw(B, H, F * L, dk, dv, frame_len=L, seed=seed, regime="slow", dtype=dtype, state_std=state_std)
    gen = torch.Generator().manual_seed(seed)
    for key in ("q", "k"):
        mag = torch.rand(B, F * L, H, 1, generator=gen) * 4.0 + 0.25
        inp[key] = (inp[key].float() * mag * np.sqrt(dk)).to(inp[key].dtype)
    inp["gamma"] = W.draw_frame_decay(B, F, H, seed=seed + 1)
    return inp


def weights(dk, seed):
    gen = torch.Generator().manual_seed(seed)
    return (torch.rand(dk, generator=gen) * 1.5 + 0.25).float(), (torch.rand(dk, generator=gen) * 1.5 + 0.25).float()


def run(inp, L, mode, wk=None, wq=None, **kw):
    d = {k: (None if v is None else v.cuda().contiguous()) for k, v in inp.items()}
    q0, k0 = d["q"].clone(), d["k"].clone()
    o, S = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], L, d.get("S_in"), return_state=True,
                     mode=mode, gamma=d["gamma"] if mode == "frame" else None, norm_keys=True, norm_queries=True,
                     k_norm_weight=None if wk is None else wk.cuda(), q_norm_weight=None if wq is None else wq.cuda(),
                     **kw)
    torch.cuda.synchronize()
    assert torch.equal(q0, d["q"]) and torch.equal(k0, d["k"])  # the inputs are not modified
    return o.double().cpu().numpy(), S.double().cpu().numpy()


def features(inp, L, wk=None, wq=None):
    kh = oracle.key_feature_map(inp["k"], frame_len=L, weight=wk)
    qh = oracle.query_feature_map(inp["q"], weight=wq)
    return qh, kh


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("weighted", [False, True])
@pytest.mark.parametrize("dk", [48, 64, 112])  # one 64-column slab, one full slab, a slab and a part
def test_prologue_framewise(dtype, weighted, dk):
    # bf16: the feature maps are applied to the kernels' staged tiles; fp32: a prologue pass
    B, H, F, L, dv = 1, 2, 4, 200, 48
    inp = raw_inputs(B, H, F, L, dk, dv, dtype, seed=51, state_std=0.1)
    wk, wq = weights(dk, 52) if weighted else (None, None)
    o, S = run(inp, L, "frame", wk, wq)
    qh, kh = features(inp, L, wk, wq)
    o_ref, S_ref = oracle.framewise(qh, kh, inp["v"], inp["gamma"], inp["beta"], inp["S_in"], frame_len=L,
                                    nthreads=NTHREADS)
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prologue_framewise_reverse_accumulate(dtype):
    B, H, F, L, dk, dv = 1, 2, 5, 64, 64, 64
    inp = raw_inputs(B, H, F, L, dk, dv, dtype, seed=57)
    wk, wq = weights(dk, 58)
    qh, kh = features(inp, L, wk, wq)
    flip = lambda x: None if x is None else torch.flip(torch.as_tensor(x), dims=[1])  # noqa: E731
    # the reversed frame-wise operator visits the frames backwards, each with its own gamma
    o_r, S_r = oracle.framewise(flip(qh), flip(kh), flip(inp["v"]), flip(inp["gamma"]), flip(inp["beta"]), None,
                                frame_len=L, nthreads=NTHREADS)
    o_ref = np.flip(o_r, axis=1)
    o0 = (torch.randn(B, F * L, H, dv, generator=torch.Generator().manual_seed(59), dtype=torch.float64)
          * 0.25 * float(np.abs(o_ref).max())).to(inp["q"].dtype)
    o, S = run(inp, L, "frame", wk, wq, o=o0.cuda(), reverse=True, accumulate=True)
    assert rel(o - o0.double().numpy(), o_ref) <= TOL[dtype]
    assert rel(S, S_r) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
def test_prologue_tokenwise(dtype, reverse):
    B, H, F, L, dk, dv = 2, 2, 3, 96, 32, 64
    inp = raw_inputs(B, H, F, L, dk, dv, dtype, seed=53, state_std=0.2)
    wk, wq = weights(dk, 54)
    o, S = run(inp, L, "token", wk, wq, reverse=reverse)
    qh, kh = features(inp, L, wk, wq)
    o_ref, S_ref = oracle.token_recurrence(qh, kh, inp["v"], inp["alpha"], inp["beta"], inp["S_in"],
                                           reverse=reverse, nthreads=NTHREADS)
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S, S_ref) <= TOL[dtype]


def test_prologue_framewise_short_clip():
    """B=1, H=20, 21 frames x 880 tokens, d = 112, bf16, raw q/k through the prologue."""
    w = W.WORKLOADS["short_clip"]
    inp = raw_inputs(w.B, w.H, w.frames, w.frame_len, w.d_k, w.d_v, "bf16", seed=W.SEEDS["short_clip"] + 5)
    o, S = run(inp, w.frame_len, "frame")
    qh, kh = features(inp, w.frame_len)
    o_ref, S_ref = oracle.framewise(qh, kh, inp["v"], inp["gamma"], inp["beta"], None, frame_len=w.frame_len,
                                    nthreads=NTHREADS)
    assert rel(o, o_ref) <= TOL["bf16"]
    assert rel(S, S_ref) <= TOL["bf16"]
