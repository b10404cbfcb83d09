"""Pins for the fp64 oracle: each test checks it against something other than
itself -- a hand-worked example, exact rational brute force, closed forms,
invariants the definition fixes, or a special case that reduces to a
textbook routine.  CPU only.

The definition pinned is the token-wise gated delta rule
``S_i = a_i S_{i-1}(I - b_i k_i k_i^T) + b_i v_i k_i^T``, ``o_i = S_i q_i``
(SANA-WM summary, paper-graph-ui, section 3.2, paragraph "Frame-wise Gated
DeltaNet (GDN)"), and the frame-wise operator of the same paragraph.
"""
import os
from fractions import Fraction

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, B, T, H, dk, dv, unit_keys=True, alpha_lo=0.5):
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit_keys:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    alpha = rng.uniform(alpha_lo, 1.0, (B, T, H))
    beta = rng.uniform(0.0, 1.0, (B, T, H))
    return q, k, v, alpha, beta


def _read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


def test_hand_worked_example():
    g = _read_golden("hand_worked_d2.txt")
    q = g["q"].reshape(1, 2, 1, 2)
    k = g["k"].reshape(1, 2, 1, 2)
    v = g["v"].reshape(1, 2, 1, 2)
    alpha = g["alpha"].reshape(1, 2, 1)
    beta = g["beta"].reshape(1, 2, 1)
    S_in = g["S_in"].reshape(1, 1, 2, 2)
    o, S = oracle.token_recurrence(q, k, v, alpha, beta, S_in)
    np.testing.assert_allclose(o.reshape(-1), g["o"], atol=1e-14)
    np.testing.assert_allclose(S.reshape(-1), g["S_out"], atol=1e-14)


def _exact_product_form(q, k, v, alpha, beta, S0):
    """S_t = S_0 F_1...F_t + sum_j beta_j v_j k_j^T F_{j+1}...F_t with
    F_i = alpha_i (I - beta_i k_i k_i^T), in exact rational arithmetic."""
    T, dk = k.shape
    dv = v.shape[1]
    Fr = lambda x: Fraction(x)  # noqa: E731  (floats here are dyadic, so exact)

    def matmul(A, Bm):
        return [[sum(A[i][m] * Bm[m][j] for m in range(len(Bm))) for j in range(len(Bm[0]))]
                for i in range(len(A))]

    Fs = []
    for i in range(T):
        a, b = Fr(alpha[i]), Fr(beta[i])
        ki = [Fr(x) for x in k[i]]
        Fs.append([[a * ((1 if r == c else 0) - b * ki[r] * ki[c]) for c in range(dk)]
                   for r in range(dk)])
    outs = []
    for t in range(T):
        P = [[Fr(x) for x in row] for row in S0]
        for i in range(t + 1):
            P = matmul(P, Fs[i])
        for j in range(t + 1):
            b = Fr(beta[j])
            term = [[b * Fr(v[j][r]) * Fr(k[j][c]) for c in range(dk)] for r in range(dv)]
            for i in range(j + 1, t + 1):
                term = matmul(term, Fs[i])
            P = [[P[r][c] + term[r][c] for c in range(dk)] for r in range(dv)]
        o = [sum(P[r][c] * Fr(q[t][c]) for c in range(dk)) for r in range(dv)]
        outs.append((o, P))
    return outs


def test_exact_rational_brute_force():
    """Tiny dyadic inputs: the fp64 oracle must equal the exact product form
    to within a few ulps."""
    rng = np.random.default_rng(7)
    T, dk, dv = 5, 3, 2
    dy = lambda shape: rng.integers(-8, 9, shape) / 8.0  # noqa: E731
    q, k, v, S0 = dy((T, dk)), dy((T, dk)), dy((T, dv)), dy((dv, dk))
    alpha = rng.integers(1, 5, T) / 4.0
    beta = rng.integers(0, 5, T) / 4.0
    o, S = oracle.token_recurrence(q[None, :, None], k[None, :, None], v[None, :, None],
                                   alpha[None, :, None], beta[None, :, None], S0[None, None])
    exact = _exact_product_form(q, k, v, alpha, beta, S0)
    for t in range(T):
        np.testing.assert_allclose(o[0, t, 0], [float(x) for x in exact[t][0]], rtol=0, atol=1e-12)
    np.testing.assert_allclose(S[0, 0], [[float(x) for x in r] for r in exact[-1][1]], atol=1e-12)


def test_product_form_brute_force_fp64():
    """Moderate sizes: explicit transition-matrix products in fp64."""
    rng = np.random.default_rng(11)
    B, T, H, dk, dv = 2, 24, 3, 8, 6
    q, k, v, alpha, beta = _rand(rng, B, T, H, dk, dv)
    S0 = rng.standard_normal((B, H, dv, dk))
    o, S = oracle.token_recurrence(q, k, v, alpha, beta, S0)
    for b in range(B):
        for h in range(H):
            F = [alpha[b, i, h] * (np.eye(dk) - beta[b, i, h] * np.outer(k[b, i, h], k[b, i, h]))
                 for i in range(T)]
            for t in range(T):
                P = S0[b, h].copy()
                for i in range(t + 1):
                    P = P @ F[i]
                for j in range(t + 1):
                    term = beta[b, j, h] * np.outer(v[b, j, h], k[b, j, h])
                    for i in range(j + 1, t + 1):
                        term = term @ F[i]
                    P = P + term
                np.testing.assert_allclose(o[b, t, h], P @ q[b, t, h], atol=1e-12)
            np.testing.assert_allclose(S[b, h], P, atol=1e-12)


def test_numpy_twin_matches_c():
    rng = np.random.default_rng(3)
    q, k, v, alpha, beta = _rand(rng, 2, 40, 3, 16, 12)
    S0 = rng.standard_normal((2, 3, 12, 16))
    o1, S1 = oracle.token_recurrence(q, k, v, alpha, beta, S0)
    o2, S2 = oracle.token_recurrence_numpy(q, k, v, alpha, beta, S0)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(S1, S2, atol=1e-12)


@settings(max_examples=40, deadline=None)
@given(B=st.integers(1, 2), T=st.integers(1, 9), H=st.integers(1, 3), dk=st.integers(1, 5),
       dv=st.integers(1, 5), seed=st.integers(0, 2 ** 31 - 1), with_state=st.booleans())
def test_numpy_twin_matches_c_any_shape(B, T, H, dk, dv, seed, with_state):
    """The C build against the numpy twin over random small shapes (layout and stride
    mistakes in the C loops show up at odd sizes)."""
    rng = np.random.default_rng(seed)
    q, k, v, alpha, beta = _rand(rng, B, T, H, dk, dv, unit_keys=False, alpha_lo=0.0)
    S0 = rng.standard_normal((B, H, dv, dk)) if with_state else None
    o1, S1 = oracle.token_recurrence(q, k, v, alpha, beta, S0, nthreads=1)
    o2, S2 = oracle.token_recurrence_numpy(q, k, v, alpha, beta, S0)
    np.testing.assert_allclose(o1, o2, rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(S1, S2, rtol=1e-10, atol=1e-10)


def test_beta0_alpha1_identity():
    """beta = 0, alpha = 1: the state never changes and o_t = S_in q_t exactly."""
    rng = np.random.default_rng(5)
    q, k, v, _, _ = _rand(rng, 1, 30, 2, 8, 8)
    S0 = rng.standard_normal((1, 2, 8, 8))
    o, S = oracle.token_recurrence(q, k, v, np.ones((1, 30, 2)), np.zeros((1, 30, 2)), S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o, np.einsum("bhvk,bthk->bthv", S0, q), atol=1e-14)


def test_beta0_closed_form_decay():
    """beta = 0: S_t = (prod_{m<=t} alpha_m) S_0, so o_t = that product times S_0 q_t."""
    rng = np.random.default_rng(6)
    q, k, v, alpha, _ = _rand(rng, 1, 20, 1, 6, 5)
    S0 = rng.standard_normal((1, 1, 5, 6))
    o, S = oracle.token_recurrence(q, k, v, alpha, np.zeros_like(alpha), S0)
    cp = np.cumprod(alpha[0, :, 0])
    for t in range(20):
        np.testing.assert_allclose(o[0, t, 0], cp[t] * S0[0, 0] @ q[0, t, 0], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(S[0, 0], cp[-1] * S0[0, 0], rtol=1e-13)


def test_orthonormal_keys_store_and_retrieve():
    """alpha = beta = 1 and orthonormal keys from S_0 = 0: S k_j = v_j exactly,
    and a read-only token (beta = 0, alpha = 1) with q = k_j returns v_j."""
    rng = np.random.default_rng(8)
    dk, dv, n = 8, 5, 8
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm.T[:n]
    vals = rng.standard_normal((n, dv))
    T = 2 * n
    k = np.zeros((1, T, 1, dk)); v = np.zeros((1, T, 1, dv)); q = np.zeros((1, T, 1, dk))
    alpha = np.ones((1, T, 1)); beta = np.ones((1, T, 1))
    k[0, :n, 0] = keys; v[0, :n, 0] = vals
    for j in range(n):                      # read-only queries
        q[0, n + j, 0] = keys[j]
        k[0, n + j, 0] = keys[(j + 1) % n]  # any unit key; beta = 0 means it is not written
        beta[0, n + j, 0] = 0.0
    o, S = oracle.token_recurrence(q, k, v, alpha, beta)
    np.testing.assert_allclose(o[0, n:, 0], vals, atol=1e-12)
    np.testing.assert_allclose(S[0, 0] @ keys.T, vals.T, atol=1e-12)


def test_delta_rule_overwrite():
    """Re-writing key k_j with a new value (alpha = beta = 1) replaces it and
    leaves the other orthonormal keys' values untouched."""
    rng = np.random.default_rng(9)
    dk, dv = 6, 4
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm.T
    vals = rng.standard_normal((dk, dv))
    new = rng.standard_normal(dv)
    k = np.concatenate([keys, keys[2:3]])[None, :, None]
    v = np.concatenate([vals, new[None]])[None, :, None]
    T = dk + 1
    o, S = oracle.token_recurrence(np.zeros((1, T, 1, dk)), k, v, np.ones((1, T, 1)), np.ones((1, T, 1)))
    expect = vals.copy(); expect[2] = new
    np.testing.assert_allclose((S[0, 0] @ keys.T).T, expect, atol=1e-12)


def test_alpha0_resets_state():
    """alpha_t = 0 forgets everything: S_t = beta_t v_t k_t^T."""
    rng = np.random.default_rng(10)
    q, k, v, alpha, beta = _rand(rng, 1, 12, 2, 7, 5)
    alpha[0, 6] = 0.0
    S0 = rng.standard_normal((1, 2, 5, 7))
    o_full, _ = oracle.token_recurrence(q, k, v, alpha, beta, S0)
    # after the reset the rest of the sequence sees only beta_6 v_6 k_6^T
    for h in range(2):
        S6 = beta[0, 6, h] * np.outer(v[0, 6, h], k[0, 6, h])
        np.testing.assert_allclose(o_full[0, 6, h], S6 @ q[0, 6, h], atol=1e-14)
    o_tail, _ = oracle.token_recurrence(q[:, 7:], k[:, 7:], v[:, 7:], alpha[:, 7:], beta[:, 7:],
                                        np.einsum("h,hv,hk->hvk", beta[0, 6], v[0, 6], k[0, 6])[None])
    np.testing.assert_allclose(o_full[:, 7:], o_tail, atol=1e-13)


def test_linearity():
    """(V, S_0) -> (O, S_T) is linear for fixed q, k, gates; O is linear in Q."""
    rng = np.random.default_rng(12)
    q, k, v1, alpha, beta = _rand(rng, 1, 25, 2, 6, 4)
    v2 = rng.standard_normal(v1.shape)
    S1 = rng.standard_normal((1, 2, 4, 6)); S2 = rng.standard_normal((1, 2, 4, 6))
    a, b = 0.7, -1.3
    oA, SA = oracle.token_recurrence(q, k, v1, alpha, beta, S1)
    oB, SB = oracle.token_recurrence(q, k, v2, alpha, beta, S2)
    oC, SC = oracle.token_recurrence(q, k, a * v1 + b * v2, alpha, beta, a * S1 + b * S2)
    np.testing.assert_allclose(oC, a * oA + b * oB, atol=1e-12)
    np.testing.assert_allclose(SC, a * SA + b * SB, atol=1e-12)
    q2 = rng.standard_normal(q.shape)
    oD, _ = oracle.token_recurrence(q2, k, v1, alpha, beta, S1)
    oE, _ = oracle.token_recurrence(a * q + b * q2, k, v1, alpha, beta, S1)
    np.testing.assert_allclose(oE, a * oA + b * oD, atol=1e-12)


def test_chained_calls_equal_one_call_and_non_expansive():
    """Single-token calls chained through S_out -> S_in equal one call, and
    with unit keys every step obeys ||S_t||_F <= ||S_{t-1}||_F + beta ||v|| ||k||
    (the transition alpha (I - beta k k^T) has spectral norm <= 1)."""
    rng = np.random.default_rng(13)
    q, k, v, alpha, beta = _rand(rng, 1, 16, 2, 6, 6)
    S = rng.standard_normal((1, 2, 6, 6))
    o_one, S_one = oracle.token_recurrence(q, k, v, alpha, beta, S)
    for t in range(16):
        sl = slice(t, t + 1)
        o_t, S_new = oracle.token_recurrence(q[:, sl], k[:, sl], v[:, sl], alpha[:, sl], beta[:, sl], S)
        np.testing.assert_allclose(o_t, o_one[:, sl], atol=1e-12)
        for h in range(2):
            bound = np.linalg.norm(S[0, h]) + beta[0, t, h] * np.linalg.norm(v[0, t, h]) * np.linalg.norm(k[0, t, h])
            assert np.linalg.norm(S_new[0, h]) <= bound + 1e-12
        S = S_new
    np.testing.assert_allclose(S, S_one, atol=1e-12)


def test_one_chunk_dense_solve_textbook():
    """One chunk evaluated through its unit-lower-triangular system, solved by
    textbook forward substitution:  with G_i = sum_{m<=i} log a_m,
    A_ij = b_i exp(G_i - G_j) k_i.k_j (j < i),
    (I + A) U = diag(b) V - diag(b e^G) K S_0^T,
    O = diag(e^G) Q S_0^T + tril(Q K^T * exp(G_i - G_j)) U,
    S_T = e^{G_T} S_0 + U^T diag(e^{G_T - G}) K."""
    rng = np.random.default_rng(14)
    T, dk, dv = 40, 8, 6
    q, k, v, alpha, beta = _rand(rng, 1, T, 1, dk, dv)
    S0 = rng.standard_normal((1, 1, dv, dk))
    o, S = oracle.token_recurrence(q, k, v, alpha, beta, S0)
    Q, K, V = q[0, :, 0], k[0, :, 0], v[0, :, 0]
    a, b, s0 = alpha[0, :, 0], beta[0, :, 0], S0[0, 0]
    G = np.cumsum(np.log(a))
    D = np.exp(G[:, None] - G[None, :])
    A = np.tril(b[:, None] * (K @ K.T) * D, -1)
    R = b[:, None] * V - (b * np.exp(G))[:, None] * (K @ s0.T)
    U = np.zeros_like(R)
    for i in range(T):  # forward substitution, row by row
        U[i] = R[i] - A[i, :i] @ U[:i]
    O = np.exp(G)[:, None] * (Q @ s0.T) + np.tril((Q @ K.T) * D) @ U
    ST = np.exp(G[-1]) * s0 + U.T @ (np.exp(G[-1] - G)[:, None] * K)
    np.testing.assert_allclose(o[0, :, 0], O, atol=1e-11)
    np.testing.assert_allclose(S[0, 0], ST, atol=1e-11)


def test_reverse_scan_is_forward_scan_of_reversed_sequence():
    rng = np.random.default_rng(15)
    q, k, v, alpha, beta = _rand(rng, 2, 18, 2, 5, 4)
    o_r, S_r = oracle.token_recurrence(q, k, v, alpha, beta, reverse=True)
    f = lambda x: x[:, ::-1].copy()  # noqa: E731
    o_f, S_f = oracle.token_recurrence(f(q), f(k), f(v), f(alpha), f(beta))
    np.testing.assert_allclose(o_r, f(o_f), atol=1e-13)
    np.testing.assert_allclose(S_r, S_f, atol=1e-13)


def test_chunk_reset_equals_independent_chunks():
    """reset_every = R: each chunk of the reversed scan starts from zero."""
    rng = np.random.default_rng(16)
    q, k, v, alpha, beta = _rand(rng, 1, 24, 2, 5, 4)
    R = 8
    o_r, _ = oracle.token_recurrence(q, k, v, alpha, beta, reverse=True, reset_every=R)
    for c in range(3):
        sl = slice(c * R, (c + 1) * R)
        o_c, _ = oracle.token_recurrence(q[:, sl], k[:, sl], v[:, sl], alpha[:, sl], beta[:, sl], reverse=True)
        np.testing.assert_allclose(o_r[:, sl], o_c, atol=1e-13)
    o_b, _ = oracle.bidirectional(q, k, v, alpha, beta, chunk_len=R)
    o_f, _ = oracle.token_recurrence(q, k, v, alpha, beta)
    np.testing.assert_allclose(o_b, o_f + o_r, atol=1e-13)


# ---------------------------------------------------------------- frame-wise operator

def test_framewise_single_token_frames_equal_tokenwise():
    """With one token per frame the frame-wise update is the token-wise one
    with alpha = gamma."""
    rng = np.random.default_rng(17)
    q, k, v, alpha, beta = _rand(rng, 2, 14, 3, 6, 5)
    S0 = rng.standard_normal((2, 3, 5, 6))
    o1, S1 = oracle.framewise(q, k, v, alpha, beta, S0, frame_len=1)
    o2, S2 = oracle.token_recurrence(q, k, v, alpha, beta, S0)
    np.testing.assert_allclose(o1, o2, atol=1e-12)
    np.testing.assert_allclose(S1, S2, atol=1e-12)


def test_framewise_orthogonal_frames_equal_tokenwise_sequence():
    """With mutually orthogonal keys inside each frame, the rank-S frame update equals
    the frame's tokens applied one by one with alpha = gamma_t at the frame's first token
    and 1 after it: the cross terms of prod_s (I - beta_s k_s k_s^T) vanish, and
    k_s^T (I - beta_s' k_s' k_s'^T) = k_s^T for s' != s.  Every token of frame t reads the
    state at the frame's end."""
    rng = np.random.default_rng(23)
    B, H, D, dv, S, F = 1, 2, 6, 5, 4, 3
    k = np.zeros((B, F * S, H, D))
    for f in range(F):
        for h in range(H):
            Qm, _ = np.linalg.qr(rng.standard_normal((D, S)))
            k[0, f * S:(f + 1) * S, h] = Qm.T
    q = rng.standard_normal((B, F * S, H, D))
    v = rng.standard_normal((B, F * S, H, dv))
    beta = rng.uniform(0, 1, (B, F * S, H))
    gamma = rng.uniform(0.3, 1.0, (B, F, H))
    S0 = rng.standard_normal((B, H, dv, D))
    o_fw, S_fw = oracle.framewise(q, k, v, gamma, beta, S0, frame_len=S)
    alpha = np.ones((B, F * S, H))
    alpha[:, ::S] = gamma
    for f in range(F):
        end = (f + 1) * S
        _, S_tok = oracle.token_recurrence(q[:, :end], k[:, :end], v[:, :end], alpha[:, :end], beta[:, :end], S0)
        for s_ in range(f * S, end):
            np.testing.assert_allclose(o_fw[0, s_], np.einsum("hvd,hd->hv", S_tok[0], q[0, s_]), atol=1e-12)
    np.testing.assert_allclose(S_fw, S_tok, atol=1e-12)


def test_framewise_orthonormal_frame_stores_values():
    """One frame of mutually orthonormal keys, beta = gamma = 1, S_0 = 0:
    every token of the frame reads S_t, and S_t k_j = v_j."""
    rng = np.random.default_rng(18)
    dk, dv = 8, 3
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm.T
    vals = rng.standard_normal((dk, dv))
    o, S = oracle.framewise(keys[None, :, None], keys[None, :, None], vals[None, :, None],
                            np.ones((1, 1, 1)), np.ones((1, dk, 1)), frame_len=dk)
    np.testing.assert_allclose(o[0, :, 0], vals, atol=1e-12)  # q = k_j reads v_j
    np.testing.assert_allclose(S[0, 0] @ keys.T, vals.T, atol=1e-12)


def test_framewise_transition_non_expansive_with_key_scaling():
    """With K_hat = ReLU(RMSNorm(K)) / sqrt(D S), tr(K_hat beta K_hat^T) <= 1
    so ||M_t||_2 <= gamma_t (SANA-WM summary, section 3.2, "Algebraic
    Stabilization for Spatial Token Explosion").  M_t is read out of the
    oracle as S_1 when S_0 = I and V = 0."""
    rng = np.random.default_rng(19)
    D, L = 16, 40
    K = rng.standard_normal((L, D))
    Kbar = np.maximum(K / np.sqrt((K * K).mean(axis=1, keepdims=True)), 0.0)
    Khat = Kbar / np.sqrt(D * L)
    beta = rng.uniform(0, 1, L)
    gamma = 0.9
    assert (beta * (Khat * Khat).sum(1)).sum() <= 1.0 + 1e-12
    _, M = oracle.framewise(np.zeros((1, L, 1, D)), Khat[None, :, None], np.zeros((1, L, 1, D)),
                            np.full((1, 1, 1), gamma), beta[None, :, None],
                            np.eye(D)[None, None], frame_len=L)
    M = M[0, 0]
    np.testing.assert_allclose(M, M.T, atol=1e-15)
    assert np.linalg.norm(M, 2) <= gamma + 1e-12
    # unscaled keys break the bound
    _, M2 = oracle.framewise(np.zeros((1, L, 1, D)), Kbar[None, :, None], np.zeros((1, L, 1, D)),
                             np.full((1, 1, 1), gamma), beta[None, :, None],
                             np.eye(D)[None, None], frame_len=L)
    assert np.linalg.norm(M2[0, 0], 2) > 1.0


def test_framewise_beta0_decay():
    rng = np.random.default_rng(20)
    q, k, v, _, _ = _rand(rng, 1, 12, 2, 4, 3)
    gamma = rng.uniform(0.5, 1.0, (1, 3, 2))
    S0 = rng.standard_normal((1, 2, 3, 4))
    o, S = oracle.framewise(q, k, v, gamma, np.zeros((1, 12, 2)), S0, frame_len=4)
    cp = np.cumprod(gamma[0], axis=0)  # [F, H]
    for t in range(12):
        for h in range(2):
            np.testing.assert_allclose(o[0, t, h], cp[t // 4, h] * S0[0, h] @ q[0, t, h], atol=1e-14)


@pytest.mark.parametrize("bad", ["T", "frame"])
def test_oracle_rejects_bad_shapes(bad):
    q = np.zeros((1, 6, 1, 2))
    if bad == "frame":
        with pytest.raises(AssertionError):
            oracle.framewise(q, q, q, np.ones((1, 1, 1)), np.ones((1, 6, 1)), frame_len=4)
    else:
        with pytest.raises(AssertionError):
            oracle.token_recurrence(q, q, q, np.ones((1, 5, 1)), np.ones((1, 6, 1)))


# ---------------------------------------------------------------- q/k prologue (feature maps)

def test_key_feature_map_constant_vector():
    """A constant positive vector has RMS equal to its value: RMSNorm maps it to ones
    (up to eps), ReLU keeps them, and the key scale makes each entry 1/sqrt(D S)."""
    D, S = 8, 5
    k = np.full((1, 1, 1, D), 3.0)
    kh = oracle.key_feature_map(k, frame_len=S, eps=0.0)
    np.testing.assert_allclose(kh, np.full_like(k, 1.0 / np.sqrt(D * S)), rtol=1e-15)
    qh = oracle.query_feature_map(-k, eps=0.0)  # all negative: ReLU zeroes it
    assert np.count_nonzero(qh) == 0


def test_feature_maps_scale_invariant_and_weighted():
    rng = np.random.default_rng(41)
    x = rng.standard_normal((2, 7, 3, 16))
    np.testing.assert_allclose(oracle.query_feature_map(5.0 * x, eps=0.0), oracle.query_feature_map(x, eps=0.0),
                               rtol=1e-13)
    w = rng.uniform(0.5, 2.0, 16)
    y = oracle.query_feature_map(x, eps=0.0)
    yw = oracle.query_feature_map(x, weight=w, eps=0.0)
    np.testing.assert_allclose(yw, y * w, rtol=1e-13)  # the weight multiplies before ReLU; w > 0 commutes
    # the RMS of the normalised vector (before ReLU) is 1: ReLU keeps sum of squares <= D
    assert (y * y).sum(-1).max() <= 16 + 1e-9
    # explicit per-entry formula on one row
    row = x[0, 0, 0]
    ref = np.maximum(row / np.sqrt(np.mean(row ** 2) + 1e-6), 0.0)
    np.testing.assert_allclose(oracle.query_feature_map(x)[0, 0, 0], ref, rtol=1e-15)


def test_key_feature_map_bounds_frame_energy():
    """The pages' bound: with beta in [0, 1], tr(K_hat^T B K_hat) = sum_s beta_s |k_hat_s|^2 <= 1
    for any frame of S keys, so every eigenvalue of I - K_hat^T B K_hat lies in [0, 1]."""
    rng = np.random.default_rng(42)
    for D, S in ((16, 40), (112, 880), (32, 1)):
        k = rng.standard_normal((1, S, 1, D)) * rng.uniform(0.1, 10.0)
        kh = oracle.key_feature_map(k, frame_len=S, eps=0.0)[0, :, 0]
        beta = rng.uniform(0, 1, S)
        A = (kh * beta[:, None]).T @ kh
        assert np.trace(A) <= 1.0 + 1e-12
        ev = np.linalg.eigvalsh(np.eye(D) - A)
        assert ev.min() >= -1e-12 and ev.max() <= 1.0 + 1e-12
