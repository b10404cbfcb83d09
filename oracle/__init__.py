"""fp64 CPU oracle for the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never calls it and
shares nothing with it: no kernels, headers, helpers, tables or pre/post
processing.  The one thing both sides share is the seeded input generator,
which lives in its own module and holds none of the method's arithmetic.

What is computed (both written from the SANA-WM summary, paper-graph-ui,
section 3.2 "Memory-Efficient Long-Context Modeling", paragraph
"Frame-wise Gated DeltaNet (GDN)"):

* ``token_recurrence`` -- the token-wise gated delta rule
  ``S_i = a_i S_{i-1} (I - b_i k_i k_i^T) + b_i v_i k_i^T``, ``o_i = S_i q_i``,
  walked one token at a time in fp64 (C, ``gdn_oracle.c``).  The chunkwise
  method the CUDA path uses reaches this result exactly up to rounding, so
  the oracle is the plain definition.
* ``framewise`` -- the frame-wise SANA-WM operator
  ``S_t = S_{t-1} M_t + U_t``, ``M_t = g_t (I - K_t B_t K_t^T)``,
  ``U_t = V_t B_t K_t^T``, ``O_t = S_t Q_t`` with M_t, U_t formed explicitly.
* ``token_recurrence_numpy`` -- a pure-Python/numpy twin of the token loop,
  for tiny cases only (cross-checks the C build and its layouts).
* ``key_feature_map`` / ``query_feature_map`` -- the q/k prologue of the same
  section's paragraph "Algebraic Stabilization for Spatial Token Explosion":
  ReLU(RMSNorm(x)) over the head dimension, keys further divided by
  sqrt(D * S).

Inputs are taken in whatever dtype they are stored in and upcast exactly to
fp64 (bf16 and fp32 both embed in fp64), so a comparison measures only the
GPU path's own error.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc -O2, OpenMP, no fast-math) next to its source."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.POINTER(ctypes.c_double)
        lib.gdn_oracle_token.argtypes = [P, P, P, P, P, P, P, P,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                         ctypes.c_longlong, ctypes.c_int]
        lib.gdn_oracle_token.restype = ctypes.c_int
        lib.gdn_oracle_framewise.argtypes = [P, P, P, P, P, P, P, P,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_longlong,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
        lib.gdn_oracle_framewise.restype = ctypes.c_int
        lib.gdn_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    """Threads an OpenMP region of the oracle uses by default."""
    return int(_load().gdn_oracle_max_threads())


def _f64(x):
    """Exact upcast to a contiguous fp64 numpy array (accepts numpy or torch)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: bf16 has no numpy dtype, upcast in torch
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def token_recurrence(q, k, v, alpha, beta, S_in=None, *, reverse=False, reset_every=0,
                     nthreads=0):
    """Token-wise gated delta rule in fp64.

    q,k: [B,T,H,d_k]; v: [B,T,H,d_v]; alpha,beta: [B,T,H]; S_in: [B,H,d_v,d_k] or None.
    ``reverse`` walks the tokens from last to first (the reversed-time scan);
    ``reset_every`` > 0 zeroes the state at each later multiple of that many
    tokens (the chunk-causal reversed scan).  Returns (o [B,T,H,d_v], S_out).
    """
    q, k, v, alpha, beta, S_in = (_f64(t) for t in (q, k, v, alpha, beta, S_in))
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    assert k.shape == (B, T, H, d_k) and v.shape == (B, T, H, d_v)
    assert alpha.shape == (B, T, H) and beta.shape == (B, T, H)
    if S_in is not None:
        assert S_in.shape == (B, H, d_v, d_k)
    o = np.zeros((B, T, H, d_v))
    S_out = np.zeros((B, H, d_v, d_k))
    rc = _load().gdn_oracle_token(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta),
                                  _ptr(S_in), _ptr(S_out), _ptr(o), B, H, T, d_k, d_v,
                                  int(bool(reverse)), int(reset_every), int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o, S_out


def framewise(q, k, v, gamma, beta, S_in=None, *, frame_len, nthreads=0):
    """Frame-wise SANA-WM operator in fp64.

    gamma: [B,F,H] per-frame decay; beta: [B,T,H] per-token gates.
    Returns (o [B,T,H,d_v], S_out [B,H,d_v,d_k]).
    """
    q, k, v, gamma, beta, S_in = (_f64(t) for t in (q, k, v, gamma, beta, S_in))
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    assert T % frame_len == 0 and gamma.shape == (B, T // frame_len, H)
    o = np.zeros((B, T, H, d_v))
    S_out = np.zeros((B, H, d_v, d_k))
    rc = _load().gdn_oracle_framewise(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(beta),
                                      _ptr(S_in), _ptr(S_out), _ptr(o), B, H, T,
                                      int(frame_len), d_k, d_v, int(nthreads))
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return o, S_out


def bidirectional(q, k, v, alpha, beta, *, chunk_len=0, S_in=None, nthreads=0):
    """Forward scan plus reversed-time scan, outputs summed (SANA-WM summary,
    section 3.2, paragraph "Bidirectional and Chunk-Causal GDN Variants").

    ``chunk_len`` > 0 gives the chunk-causal form: the forward scan stays
    global, the reversed scan restarts from zero at each chunk boundary.
    Returns (o, S_out of the forward scan).
    """
    o_f, S_f = token_recurrence(q, k, v, alpha, beta, S_in, nthreads=nthreads)
    o_r, _ = token_recurrence(q, k, v, alpha, beta, None, reverse=True,
                              reset_every=chunk_len, nthreads=nthreads)
    return o_f + o_r, S_f


def key_feature_map(k, *, frame_len, weight=None, eps=1e-6):
    """Keys of the frame-wise operator (SANA-WM summary, "Memory-Efficient
    Long-Context Modeling (Section 3.2)", paragraph "Algebraic Stabilization
    for Spatial Token Explosion"): k_bar = ReLU(RMSNorm(k)) over the head
    dimension D, then k_hat = k_bar / sqrt(D * S) with S = frame_len tokens.
    RMSNorm(x) = x / sqrt(mean(x^2) + eps) * weight (weight = ones if None).
    In fp64; returns a numpy array of k's shape."""
    y = _rms_relu(k, weight, eps)
    return y / np.sqrt(y.shape[-1] * float(frame_len))


def query_feature_map(q, *, weight=None, eps=1e-6):
    """Queries: q_hat = ReLU(RMSNorm(q)) (the keys' feature map without the
    1/sqrt(D*S) scale, which the same paragraph applies to keys only)."""
    return _rms_relu(q, weight, eps)


def _rms_relu(x, weight, eps):
    x = _f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    y = x / np.sqrt(ms + eps)
    if weight is not None:
        y = y * _f64(weight)
    return np.maximum(y, 0.0)


def token_recurrence_numpy(q, k, v, alpha, beta, S_in=None):
    """Pure numpy twin of ``token_recurrence`` (forward only); tiny cases only."""
    q, k, v, alpha, beta, S_in = (_f64(t) for t in (q, k, v, alpha, beta, S_in))
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    o = np.zeros((B, T, H, d_v))
    S_out = np.zeros((B, H, d_v, d_k))
    for b in range(B):
        for h in range(H):
            S = np.zeros((d_v, d_k)) if S_in is None else S_in[b, h].copy()
            for t in range(T):
                kt, vt, qt = k[b, t, h], v[b, t, h], q[b, t, h]
                a, be = alpha[b, t, h], beta[b, t, h]
                S = a * S @ (np.eye(d_k) - be * np.outer(kt, kt)) + be * np.outer(vt, kt)
                o[b, t, h] = S @ qt
            S_out[b, h] = S
    return o, S_out
