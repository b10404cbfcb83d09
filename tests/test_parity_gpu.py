"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Metric: max|x - x_ref| / max|x_ref| over the compared elements, for o and
for S_out.  Bars: 1e-5 for the fp32 path (fp32 q/k/v/o), 2e-2 for bf16
inputs with an fp32 state.  Inputs are the seeded synthetic workloads; both
gate regimes run ("lit": alpha = exp(-softplus(z+2)), "slow": z-4).
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


def dev(inp):
    return {k: (None if v is None else v.cuda().contiguous()) for k, v in inp.items()}


def accumulate_offset(o_ref, dtype, seed):
    """What o holds before an accumulating call: values exactly representable in the
    output dtype, a quarter of the result's scale.  o then stores round(o + result) once,
    so o - offset differs from the result by one rounding at |o + offset| <= 1.25 max|o|,
    the same order as the rounding of a plain call's output."""
    gen = torch.Generator().manual_seed(1234 + seed)
    scale = 0.25 * float(np.abs(o_ref).max())
    return (torch.randn(o_ref.shape, generator=gen, dtype=torch.float64) * scale).to(dtype)


def gpu_fwd(inp, frame_len, S_in=None, **kw):
    d = dev(inp)
    S = None if S_in is None else S_in.cuda().contiguous()
    o, S_out = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], frame_len, S,
                         return_state=True, **kw)
    torch.cuda.synchronize()
    return o.double().cpu().numpy(), S_out.double().cpu().numpy()


def ora(inp, S_in=None, **kw):
    return oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                   S_in, nthreads=NTHREADS, **kw)


@pytest.mark.parametrize("regime", ["lit", "slow"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tiny(regime, dtype):
    inp = W.draw(1, 2, 256, 64, 64, frame_len=64, seed=W.SEEDS["tiny"], regime=regime, dtype=dtype)
    o, S = gpu_fwd(inp, 64)
    o_ref, S_ref = ora(inp)
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S, S_ref) <= TOL[dtype]


# ragged frames and head dims, several 32/128-row blocks plus a tail
CASES = [
    # B, H, frames, L, dk, dv, dtype
    (2, 3, 3, 100, 48, 80, "f32"),
    (1, 2, 2, 300, 128, 64, "f32"),
    (1, 1, 5, 17, 16, 128, "f32"),
    (1, 2, 6, 1, 32, 32, "f32"),
    (1, 2, 2, 880, 112, 112, "bf16"),
    (2, 2, 3, 200, 64, 96, "bf16"),
    (1, 1, 2, 129, 128, 128, "bf16"),
    (1, 1, 1, 4096, 64, 64, "bf16"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dF%dL%d_dk%d_dv%d_%s" % c)
@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_ragged(case, regime):
    B, H, F, L, dk, dv, dtype = case
    inp = W.draw(B, H, F * L, dk, dv, frame_len=L, seed=77, regime=regime, dtype=dtype, state_std=0.1)
    o, S = gpu_fwd(inp, L, S_in=inp["S_in"])
    o_ref, S_ref = ora(inp, inp["S_in"])
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_state_in_place(dtype):
    inp = W.draw(1, 3, 2 * 96, 64, 64, frame_len=96, seed=5, regime="slow", dtype=dtype, state_std=0.5)
    d = dev(inp)
    S = d["S_in"].clone()
    o, S2 = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 96, S, S_out=S)
    torch.cuda.synchronize()
    assert S2.data_ptr() == S.data_ptr()
    o_ref, S_ref = ora(inp, inp["S_in"])
    assert rel(o.double().cpu(), o_ref) <= TOL[dtype]
    assert rel(S.double().cpu(), S_ref) <= TOL[dtype]


def test_empty_sequences():
    x = torch.zeros(1, 0, 2, 32, device="cuda")
    a = torch.zeros(1, 0, 2, device="cuda")
    S_in = torch.randn(1, 2, 32, 32, device="cuda")
    o, S = g.gdn_fwd(x, x, x, a, a, 16, S_in, return_state=True)
    torch.cuda.synchronize()
    assert o.shape == (1, 0, 2, 32)
    assert torch.equal(S, S_in)
    o, S = g.gdn_fwd(x, x, x, a, a, 16, None, return_state=True)
    assert torch.count_nonzero(S) == 0
    z = torch.zeros(0, 64, 2, 32, device="cuda")
    g.gdn_fwd(z, z, z, torch.zeros(0, 64, 2, device="cuda"), torch.zeros(0, 64, 2, device="cuda"), 16)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_gate_edge_cases(dtype):
    """alpha = 0 (full reset) mid-frame and at a frame start, beta = 0 tokens, alpha = 1 runs."""
    inp = W.draw(1, 2, 3 * 64, 32, 32, frame_len=64, seed=9, regime="slow", dtype=dtype, state_std=0.3)
    inp["alpha"][0, 10] = 0.0
    inp["alpha"][0, 64] = 0.0
    inp["alpha"][0, 100:140] = 1.0
    inp["beta"][0, 20:30] = 0.0
    inp["beta"][0, 150] = 1.0
    o, S = gpu_fwd(inp, 64, S_in=inp["S_in"])
    o_ref, S_ref = ora(inp, inp["S_in"])
    assert np.isfinite(o).all() and np.isfinite(S).all()
    assert rel(o, o_ref) <= TOL[dtype]
    assert rel(S, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("chunk", [0, 2])
def test_reverse_and_bidirectional(dtype, chunk):
    L = 48
    inp = W.draw(2, 2, 6 * L, 32, 48, frame_len=L, seed=21, regime="slow", dtype=dtype, state_std=0.2)
    d = dev(inp)
    o_r, S_r = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], L, d["S_in"], return_state=True,
                         reverse=True, reset_every=chunk * L)
    o_ref, S_ref = ora(inp, inp["S_in"], reverse=True, reset_every=chunk * L)
    assert rel(o_r.double().cpu(), o_ref) <= TOL[dtype]
    assert rel(S_r.double().cpu(), S_ref) <= TOL[dtype]
    o_b, _ = g.bidirectional(d["q"], d["k"], d["v"], d["alpha"], d["beta"], L, chunk_len=chunk * L)
    ob_ref, _ = oracle.bidirectional(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], chunk_len=chunk * L)
    assert rel(o_b.double().cpu(), ob_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reverse_reset_not_dividing_length(dtype):
    # 5 frames, state restarting every 2 frames counted from token 0: the reversed scan's
    # restarts do not line up with its own start
    L = 64
    inp = W.draw(1, 3, 5 * L, 48, 32, frame_len=L, seed=23, regime="slow", dtype=dtype, state_std=0.2)
    d = dev(inp)
    o_ref, S_ref = ora(inp, inp["S_in"], reverse=True, reset_every=2 * L)
    c = accumulate_offset(o_ref, d["q"].dtype, seed=1)  # accumulate into a non-zero o
    o_r, S_r = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], L, d["S_in"], return_state=True,
                         reverse=True, reset_every=2 * L, o=c.cuda(), accumulate=True)
    assert rel(o_r.double().cpu() - c.double(), o_ref) <= TOL[dtype]
    assert rel(S_r.double().cpu(), S_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_reverse_accumulate_in_caller_workspace(dtype):
    # a workspace of gdn_workspace_bytes serves the largest case, a reversed accumulating call
    B, H, L, F, dk, dv = 1, 2, 64, 3, 32, 48
    inp = W.draw(B, H, F * L, dk, dv, frame_len=L, seed=25, regime="slow", dtype=dtype)
    d = dev(inp)
    ws = torch.empty(g.workspace_bytes(B, H, F * L, L, dk, dv, dtype), dtype=torch.uint8, device="cuda")
    o_ref, _ = ora(inp, None, reverse=True)
    c = accumulate_offset(o_ref, d["q"].dtype, seed=2)
    o_r, _ = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], L, None, o=c.cuda(), reverse=True,
                       accumulate=True, workspace=ws)
    torch.cuda.synchronize()
    assert rel(o_r.double().cpu() - c.double(), o_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_status_word_reports_no_timeout(dtype):
    # status_dev is written in stream order: 0 after a pass whose device waits all completed
    inp = W.draw(1, 2, 2 * 64, 32, 32, frame_len=64, seed=27, regime="slow", dtype=dtype)
    d = dev(inp)
    st = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    o, _ = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 64, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    o_ref, _ = ora(inp)
    assert rel(o.double().cpu(), o_ref) <= TOL[dtype]
    st.fill_(7)
    z = d["q"][:, :0].contiguous()
    g.gdn_fwd(z, z, z, d["alpha"][:, :0].contiguous(), d["beta"][:, :0].contiguous(), 64, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_step_chain_equals_single_call(dtype):
    L = 80
    inp = W.draw(2, 3, 7 * L, 64, 64, frame_len=L, seed=31, regime="slow", dtype=dtype, state_std=0.1)
    d = dev(inp)
    o_full, S_full = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], L, d["S_in"], return_state=True)
    S = d["S_in"].clone()
    outs = []
    for f0, f1 in [(0, 1), (1, 4), (4, 6), (6, 7)]:
        sl = slice(f0 * L, f1 * L)
        args = [d[n][:, sl].contiguous() for n in ("q", "k", "v", "alpha", "beta")]
        o, _ = g.gdn_step(*args, L, S, S_out=S)
        outs.append(o)
    torch.cuda.synchronize()
    o_chain = torch.cat(outs, dim=1)
    o_ref, S_ref = ora(inp, inp["S_in"])
    assert rel(o_chain.double().cpu(), o_ref) <= TOL[dtype]
    assert rel(S.double().cpu(), S_ref) <= TOL[dtype]
    # chained calls and one call agree to rounding
    assert rel(o_chain.double().cpu(), o_full.double().cpu()) <= TOL[dtype]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_host_entry_matches_device_call(dtype):
    # gdn_fwd_host runs the same kernels on copies of the host buffers
    inp = W.draw(1, 3, 2 * 200, 64, 96, frame_len=200, seed=5, regime="slow", dtype=dtype, state_std=0.1)
    o_dev, S_dev = gpu_fwd(inp, 200, S_in=inp["S_in"])
    h = {k: (None if v is None else v.contiguous().pin_memory()) for k, v in inp.items()}
    o_h, S_h = g.gdn_fwd_host(h["q"], h["k"], h["v"], h["alpha"], h["beta"], 200, h["S_in"], return_state=True)
    assert np.array_equal(o_h.double().numpy(), o_dev) and np.array_equal(S_h.double().numpy(), S_dev)
    o_ref, S_ref = ora(inp, inp["S_in"])
    assert rel(o_h.double().numpy(), o_ref) <= TOL[dtype]


def test_deterministic():
    inp = W.draw(1, 4, 2 * 880, 112, 112, frame_len=880, seed=3, regime="slow", dtype="bf16")
    d = dev(inp)
    o1, S1 = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 880, None, return_state=True)
    o2, S2 = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 880, None, return_state=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_caller_workspace_and_finite_check():
    inp = W.draw(1, 2, 2 * 128, 64, 64, frame_len=128, seed=4, regime="lit", dtype="bf16")
    d = dev(inp)
    nbytes = g.workspace_bytes(1, 2, 256, 128, 64, 64, "bf16")
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    o1, _ = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 128, workspace=ws)
    o2, _ = g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 128, check_finite=True)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)
    with pytest.raises(g.GdnError) as ei:
        g.gdn_fwd(d["q"], d["k"], d["v"], d["alpha"], d["beta"], 128, workspace=ws[: nbytes // 2])
    assert ei.value.name == "GDN_ERR_NO_MEMORY"
    v = d["v"].clone()
    v[0, 5, 1, 3] = float("nan")
    with pytest.raises(g.GdnError) as ei:
        g.gdn_fwd(d["q"], d["k"], v, d["alpha"], d["beta"], 128, check_finite=True)
    assert ei.value.name == "GDN_ERR_NONFINITE"


# ------------------------------------------------------------ the named workloads

@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_short_clip(regime):
    w = W.WORKLOADS["short_clip"]
    inp = W.make_inputs(w, regime)
    o, S = gpu_fwd(inp, w.frame_len)
    heads = [0, 7, 19]
    sub = {k: (v[:, :, heads] if v is not None and v.dim() >= 3 else v) for k, v in inp.items()}
    o_ref, S_ref = ora(sub)
    assert rel(o[:, :, heads], o_ref) <= TOL["bf16"]
    assert rel(S[:, heads], S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_minute_sampled_heads(regime):
    """Full 106,480-token pass (the benchmarked launch); two heads checked
    against the oracle over every token."""
    w = W.WORKLOADS["minute"]
    inp = W.make_inputs(w, regime)
    o, S = gpu_fwd(inp, w.frame_len)
    # the full-size launch is bit-reproducible (no race between the pipelined stages)
    o2, S2 = gpu_fwd(inp, w.frame_len)
    assert np.array_equal(o, o2) and np.array_equal(S, S2)
    heads = [3, 16]
    sub = {k: (v[:, :, heads] if v is not None and v.dim() >= 3 else v) for k, v in inp.items()}
    o_ref, S_ref = ora(sub)
    assert rel(o[:, :, heads], o_ref) <= TOL["bf16"]
    assert rel(S[:, heads], S_ref) <= TOL["bf16"]
    assert np.isfinite(o).all()


@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_ar_rollout(regime):
    """40 chained gdn_step calls (4 + 39 x 3 frames) with per-frame alpha,
    state carried S_out -> S_in; two (b, h) chains checked over all 121 frames."""
    w = W.WORKLOADS["ar_rollout"]
    inp = W.make_inputs(w, regime)
    d = dev(inp)
    L = w.frame_len
    S = torch.zeros(w.B, w.H, w.d_v, w.d_k, device="cuda")
    o_all = torch.empty_like(d["v"])
    f0 = 0
    for nf in w.calls:
        sl = slice(f0 * L, (f0 + nf) * L)
        args = [d[n][:, sl].contiguous() for n in ("q", "k", "v", "alpha", "beta")]
        o, _ = g.gdn_step(*args, L, S, S_out=S)
        o_all[:, sl] = o
        f0 += nf
    torch.cuda.synchronize()
    assert f0 == w.frames
    for b, h in [(0, 5), (1, 12)]:
        sub = {k: (v[b:b + 1, :, h:h + 1] if v is not None and v.dim() >= 3 else v) for k, v in inp.items()}
        o_ref, S_ref = ora(sub)
        assert rel(o_all[b:b + 1, :, h:h + 1].double().cpu(), o_ref) <= TOL["bf16"]
        assert rel(S[b:b + 1, h:h + 1].double().cpu(), S_ref) <= TOL["bf16"]


@pytest.mark.parametrize("regime", ["lit", "slow"])
def test_decode_calls(regime):
    """Streaming decode: B=8, one 880-token frame per call, preloaded random
    state; the first three carried calls checked on every chain."""
    w = W.WORKLOADS["decode"]
    S = None
    S_ref = None
    for c in range(3):
        inp = W.make_inputs(w, regime, call=c)
        if c == 0:
            S = inp["S_in"].cuda()
            S_ref = inp["S_in"].double().numpy()
        d = dev(inp)
        o, _ = g.gdn_step(d["q"], d["k"], d["v"], d["alpha"], d["beta"], w.frame_len, S, S_out=S)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.token_recurrence(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                               S_ref, nthreads=NTHREADS)
        assert rel(o.double().cpu(), o_ref) <= TOL["bf16"]
        assert rel(S.double().cpu(), S_ref) <= TOL["bf16"]
