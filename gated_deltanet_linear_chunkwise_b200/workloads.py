"""Named workloads and their seeded synthetic inputs.

This module only draws numbers: it holds none of the gated delta rule's
arithmetic, so the CUDA path and the fp64 oracle can both take their inputs
from it.

Shapes follow the SANA-WM pages: a 704x1280 clip is 22x40 = 880 latent
tokens per frame and a minute is 121 latent frames, 106,480 tokens
(SANA-WM teardown, thesatyajit, section "Why a minute is hard: count the
tokens"); d_model 2240 split into 20 heads of 112 (same page, section "The
linear part: a gated delta rule, one frame per step": a 112x112 state per
head, 20 heads).

Recipe (seeded numpy ``default_rng``; every draw in fp32, in this order):
q, k, v, z_beta, z_alpha, S_in.

* q, k ~ N(0,1), L2-normalised per token in fp64, then cast to the stored dtype.
* v ~ N(0,1).
* beta = sigmoid(z_beta), z_beta ~ N(0,1).
* alpha = exp(-softplus(z_alpha + c)), z_alpha ~ N(0,1); c = +2 for the
  gate regime ``"lit"`` (the distribution formula as written: median decay
  ~0.12 per token) and c = -4 for ``"slow"`` (median ~0.98, the ~0.9-1 decay
  the workload description glosses it as).  Per-frame gating draws z_alpha
  once per (batch, frame, head) and repeats it over the frame's tokens.
* S_in (only where the workload preloads a state) = std * N(0,1).
"""
from __future__ import annotations

import dataclasses

import numpy as np

FRAME_TOKENS = 880  # 22 x 40 latent tokens per 704x1280 frame
MINUTE_FRAMES = 121  # 961 raw frames -> 121 latent frames

GATE_SHIFT = {"lit": 2.0, "slow": -4.0}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    frames: int
    frame_len: int
    d_k: int
    d_v: int
    dtype: str  # "bf16" or "f32": the stored dtype of q, k, v and o
    per_frame_alpha: bool = False
    calls: tuple = ()  # frames per call for multi-call rollouts; () = one call
    state_std: float = 0.0  # > 0: preload S_in ~ state_std * N(0,1)
    fresh_per_call: bool = False  # each call draws its own q/k/v/alpha/beta

    @property
    def T(self) -> int:
        return self.frames * self.frame_len


WORKLOADS = {
    # tiny oracle case: 4 frames x 64 tokens, fp32
    "tiny": Workload("tiny", B=1, H=2, frames=4, frame_len=64, d_k=64, d_v=64, dtype="f32"),
    # short clip: 21 latent frames x 880 tokens
    "short_clip": Workload("short_clip", B=1, H=20, frames=21, frame_len=FRAME_TOKENS,
                           d_k=112, d_v=112, dtype="bf16"),
    # minute-scale pass: 121 latent frames x 880 tokens = 106,480 tokens
    "minute": Workload("minute", B=1, H=20, frames=MINUTE_FRAMES, frame_len=FRAME_TOKENS,
                       d_k=112, d_v=112, dtype="bf16"),
    # chunk-causal rollout: 40 calls of 3 frames (first call 4), state carried
    "ar_rollout": Workload("ar_rollout", B=2, H=20, frames=MINUTE_FRAMES, frame_len=FRAME_TOKENS,
                           d_k=112, d_v=112, dtype="bf16", per_frame_alpha=True,
                           calls=(4,) + (3,) * 39),
    # streaming decode: one new frame per call, 100 calls, preloaded random state
    "decode": Workload("decode", B=8, H=20, frames=100, frame_len=FRAME_TOKENS,
                       d_k=112, d_v=112, dtype="bf16", calls=(1,) * 100,
                       state_std=0.02, fresh_per_call=True),
}

# seed = workload index + 1000
SEEDS = {name: 1000 + i for i, name in enumerate(WORKLOADS)}


def _normalise_rows(x: np.ndarray, chunk: int = 1 << 20) -> np.ndarray:
    """L2-normalise the last axis in fp64, chunk by chunk, back to fp32."""
    flat = x.reshape(-1, x.shape[-1])
    out = np.empty_like(flat)
    for s in range(0, flat.shape[0], chunk):
        blk = flat[s:s + chunk].astype(np.float64)
        blk /= np.sqrt((blk * blk).sum(axis=1, keepdims=True))
        out[s:s + chunk] = blk.astype(np.float32)
    return out.reshape(x.shape)


def draw(B, H, T, d_k, d_v, *, frame_len, seed, regime="lit", per_frame_alpha=False,
         state_std=0.0, dtype="bf16"):
    """Draw one call's inputs.  Returns a dict of torch CPU tensors:
    q,k [B,T,H,d_k] and v [B,T,H,d_v] in the stored dtype, alpha/beta
    [B,T,H] fp32, S_in [B,H,d_v,d_k] fp32 or None."""
    import torch

    rng = np.random.default_rng(seed)
    shift = GATE_SHIFT[regime]
    q = rng.standard_normal((B, T, H, d_k), dtype=np.float32)
    k = rng.standard_normal((B, T, H, d_k), dtype=np.float32)
    v = rng.standard_normal((B, T, H, d_v), dtype=np.float32)
    z_beta = rng.standard_normal((B, T, H), dtype=np.float32)
    if per_frame_alpha:
        z_alpha = rng.standard_normal((B, T // frame_len, H), dtype=np.float32)
        z_alpha = np.repeat(z_alpha, frame_len, axis=1)
    else:
        z_alpha = rng.standard_normal((B, T, H), dtype=np.float32)
    S_in = None
    if state_std > 0:
        S_in = (state_std * rng.standard_normal((B, H, d_v, d_k), dtype=np.float32)).astype(np.float32)

    q = _normalise_rows(q)
    k = _normalise_rows(k)
    beta = (1.0 / (1.0 + np.exp(-z_beta.astype(np.float64)))).astype(np.float32)
    alpha = np.exp(-np.logaddexp(0.0, z_alpha.astype(np.float64) + shift)).astype(np.float32)

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {
        "q": torch.from_numpy(q).to(tdt),
        "k": torch.from_numpy(k).to(tdt),
        "v": torch.from_numpy(v).to(tdt),
        "alpha": torch.from_numpy(alpha),
        "beta": torch.from_numpy(beta),
        "S_in": None if S_in is None else torch.from_numpy(S_in),
    }
    return out


def draw_frame_decay(B, F, H, *, seed, regime="slow"):
    """Per-frame decays gamma [B, F, H] fp32 for the frame-wise operator, drawn
    with the alpha recipe (exp(-softplus(z + c)), z ~ N(0,1)) once per (batch,
    frame, head) from their own seeded stream."""
    import torch

    rng = np.random.default_rng(seed)
    z = rng.standard_normal((B, F, H), dtype=np.float32)
    gamma = np.exp(-np.logaddexp(0.0, z.astype(np.float64) + GATE_SHIFT[regime])).astype(np.float32)
    return torch.from_numpy(gamma)


def make_inputs(w: Workload | str, regime="lit", *, seed=None, call=None, frames=None):
    """Inputs for a named workload.

    For a fresh-per-call workload, ``call`` selects which call's draw is made
    (seeded by (seed, call)); the preloaded state is part of call 0's draw.
    ``frames`` overrides the frame count (a truncated sample of the same
    recipe, for bounded CPU runs).
    """
    if isinstance(w, str):
        w = WORKLOADS[w]
    seed = SEEDS[w.name] if seed is None else seed
    n_frames = w.frames if frames is None else frames
    if w.fresh_per_call:
        c = 0 if call is None else int(call)
        n_frames = w.calls[c] if frames is None else frames
        seed = [seed, c]
    return draw(w.B, w.H, n_frames * w.frame_len, w.d_k, w.d_v, frame_len=w.frame_len,
                seed=seed, regime=regime, per_frame_alpha=w.per_frame_alpha,
                state_std=(w.state_std if (not w.fresh_per_call or not call) else 0.0),
                dtype=w.dtype)
