"""Parity of the frame-wise operator (``mode="frame"``) through the C ABI
with the fp64 oracle's ``framewise`` (SANA-WM summary, "Memory-Efficient
Long-Context Modeling (Section 3.2)", paragraph "Adaptation to video:
frame-wise recurrence").

Metric and bars as for the token-wise path: max|x - x_ref| / max|x_ref|,
1e-5 for fp32 q/k/v/o, 2e-2 for bf16.  Keys are the workload's unit keys
scaled by 1/sqrt(frame_len), so sum_s beta_s |k_s|^2 <= 1 and every M_t is
non-expansive (the stabilisation the same section derives); without it the
state grows geometrically over frames.
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


def inputs(B, H, F, L, dk, dv, dtype, seed, regime="slow", state_std=0.0):
    inp = W.draw(B, H, F * L, dk, dv, frame_len=L, seed=seed, regime=regime, dtype=dtype,
                 state_std=state_std)
    inp["k"] = (inp["k"].float() / np.sqrt(L)).to(inp["k"].dtype)
    inp["gamma"] = W.draw_frame_decay(B, F, H, seed=seed + 1, regime=regime)
    return inp


def gpu(inp, L, S_in=None, o=None, **kw):
    d = {k: (None if v is None else v.cuda().contiguous()) for k, v in inp.items()}
    S = None if S_in is None else S_in.cuda().contiguous()
    o_dev = None if o is None else o.cuda().contiguous()
    out, S_out = g.gdn_fwd(d["q"], d["k"], d["v"], None, d["beta"], L, S, o=o_dev, return_state=True,
                           mode="frame", gamma=d["gamma"], **kw)
    torch.cuda.synchronize()
    return out.double().cpu().numpy(), S_out.double().cpu().numpy()


def ref(inp, L, S_in=None):
    return oracle.framewise(inp["q"], inp["k"], inp["v"], inp["gamma"], inp["beta"], S_in, frame_len=L,
                            nthreads=NTHREADS)


def flip(inp):
    """Token- and frame-reversed copy: the reversed scan is the forward one on it."""
    out = dict(inp)
    for key in ("q", "k", "v", "beta"):
        out[key] = torch.flip(inp[key], dims=[1])
    out["gamma"] = torch.flip(inp["gamma"], dims=[1])
    return out


CASES = [
    # B, H, frames, L, dk, dv, dtype
    (1, 2, 4, 64, 64, 64, "f32"),
    (2, 3, 3, 100, 48, 80, "f32"),
    (1, 2, 6, 1, 32, 32, "f32"),
    (1, 1, 5, 17, 16, 128, "f32"),
    (1, 2, 3, 880, 112, 112, "bf16"),
    (2, 2, 3, 200, 64, 96, "bf16"),
    (1, 1, 2, 129, 128, 128, "bf16"),
    (1, 1, 2, 4096, 64, 64, "bf16"),
    (1, 2, 4, 40, 16, 16, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dF%dL%d_dk%d_dv%d_%s" % c)
@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_framewise_parity(case, regime):
    B, H, F, L, dk, dv, dtype = case
    inp = inputs(B, H, F, L, dk, dv, dtype, seed=31, regime=regime, state_std=0.1)
    o, S = gpu(inp, L, S_in=inp["S_in"])
    o_ref, S_ref = ref(inp, L, inp["S_in"])
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_framewise_reverse_and_accumulate(dtype):
    B, H, F, L, dk, dv = 1, 2, 5, 96, 64, 48
    inp = inputs(B, H, F, L, dk, dv, dtype, seed=32)
    o_r, S_r = ref(flip(inp), L)
    o_ref = np.flip(o_r, axis=1)
    # o holds values exactly representable in its dtype, a quarter of the result's scale,
    # so o - o0 carries one rounding at |o0 + result|, the order of a plain call's
    o0 = (torch.randn(B, F * L, H, dv, generator=torch.Generator().manual_seed(32), dtype=torch.float64)
          * 0.25 * float(np.abs(o_ref).max())).to(inp["q"].dtype)
    o, S = gpu(inp, L, o=o0.clone(), reverse=True, accumulate=True)
    assert rel(o - o0.double().numpy(), o_ref) <= TOL[dtype]
    assert rel(S, S_r) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("reverse", [False, True])
def test_framewise_chunk_reset(dtype, reverse):
    # the state restarts from zero at every boundary of 2 frames (counted from token 0)
    B, H, F, L, dk, dv = 1, 2, 6, 48, 32, 32
    inp = inputs(B, H, F, L, dk, dv, dtype, seed=33, state_std=0.2)
    o, S = gpu(inp, L, S_in=inp["S_in"], reverse=reverse, reset_every=2 * L)
    src = flip(inp) if reverse else inp
    o_ref = np.zeros_like(o)
    S_ref = None
    for c in range(F // 2):  # chunks in scan order; the first one keeps S_in
        sl = slice(2 * c * L, 2 * (c + 1) * L)
        part = {k: src[k][:, sl] for k in ("q", "k", "v", "beta")}
        part["gamma"] = src["gamma"][:, 2 * c:2 * c + 2]
        oc, S_ref = ref(part, L, inp["S_in"] if c == 0 else None)
        o_ref[:, sl] = oc
    if reverse:
        o_ref = np.flip(o_ref, axis=1)
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S, S_ref) <= TOL[dtype]


def test_framewise_state_carry_matches_one_call():
    # two calls with the state carried equal one call over all frames
    B, H, F, L, dk, dv = 2, 2, 4, 128, 64, 64
    inp = inputs(B, H, F, L, dk, dv, "bf16", seed=34, state_std=0.1)
    half = {k: inp[k][:, :2 * L] for k in ("q", "k", "v", "beta")}
    half["gamma"] = inp["gamma"][:, :2]
    rest = {k: inp[k][:, 2 * L:] for k in ("q", "k", "v", "beta")}
    rest["gamma"] = inp["gamma"][:, 2:]
    o1, S1 = gpu(half, L, S_in=inp["S_in"])
    o2, S2 = gpu(rest, L, S_in=torch.from_numpy(S1).float())
    o_ref, S_ref = ref(inp, L, inp["S_in"])
    assert rel(np.concatenate([o1, o2], axis=1), o_ref) <= TOL["bf16"]
    assert rel(S2, S_ref) <= TOL["bf16"]


def test_framewise_single_token_frames_equal_tokenwise_gpu():
    # frames of one token: the frame-wise operator is the token-wise rule with alpha = gamma
    B, H, T, d = 1, 2, 48, 32
    inp = inputs(B, H, T, 1, d, d, "f32", seed=35, state_std=0.1)
    alpha = inp["gamma"].clone()  # [B, T, H]
    o_f, S_f = gpu(inp, 1, S_in=inp["S_in"])
    d_ = {k: (None if v is None else v.cuda()) for k, v in inp.items()}
    o_t, S_t = g.gdn_fwd(d_["q"], d_["k"], d_["v"], alpha.cuda(), d_["beta"], 1, d_["S_in"], return_state=True)
    torch.cuda.synchronize()
    assert rel(o_f, o_t.double().cpu()) <= TOL["f32"]
    assert rel(S_f, S_t.double().cpu()) <= TOL["f32"]


def test_framewise_short_clip_full_size():
    """B=1, H=20, 21 frames x 880 tokens, d = 112, bf16: every element against the oracle."""
    w = W.WORKLOADS["short_clip"]
    inp = inputs(w.B, w.H, w.frames, w.frame_len, w.d_k, w.d_v, "bf16", seed=W.SEEDS["short_clip"])
    o, S = gpu(inp, w.frame_len)
    o_ref, S_ref = ref(inp, w.frame_len)
    assert rel(o, o_ref) <= TOL["bf16"]
    assert rel(S, S_ref) <= TOL["bf16"]
    # the same call twice gives the same bits
    o2, _ = gpu(inp, w.frame_len)
    assert np.array_equal(o, o2)


def test_framewise_gamma_zero_resets():
    # gamma = 0 drops everything before the frame: the state after it is U_t alone
    B, H, F, L, d = 1, 1, 3, 32, 32
    inp = inputs(B, H, F, L, d, d, "f32", seed=36, state_std=0.5)
    inp["gamma"][0, 1, 0] = 0.0
    o, S = gpu(inp, L, S_in=inp["S_in"])
    o_ref, S_ref = ref(inp, L, inp["S_in"])
    assert rel(o, o_ref) <= TOL["f32"]
    assert rel(S, S_ref) <= TOL["f32"]
    # the last two frames do not depend on S_in
    o0, _ = gpu(inp, L, S_in=torch.zeros_like(inp["S_in"]))
    assert rel(o[:, L:], o0[:, L:]) <= TOL["f32"]
