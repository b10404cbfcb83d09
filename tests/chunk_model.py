"""fp64 numpy model of the chunk = frame algebra the CUDA kernels evaluate.

Test-side only, and NOT the oracle: it restates the kernels' decomposition so
that the derivation can be checked against the oracle on the CPU, and so the
rounding points of the bf16 tensor-core path can be simulated at full frame
size.  Per chain and frame (G = inclusive prefix of log alpha in the frame):

  (I + A)[Ub | W] = [diag(beta) V | diag(beta e^G) K],
      A_ij = beta_i e^{G_i - G_j} k_i.k_j  (j < i), blocked forward substitution
  U = Ub - W Sig,  M = e^{G_L} I - Kt^T W,  N = Kt^T Ub,  Kt = diag(e^{G_L - G}) K
  O = diag(e^G) Q Sig + tril_incl(Q K^T o e^{G_i - G_j}) U,  Sig <- M Sig + N
with Sig = S^T.
"""
import numpy as np

LOG_FLOOR = -200.0


def _bf16(x):
    """Round to bf16 (nearest-even) and back, in numpy."""
    x = np.asarray(x, dtype=np.float32)
    b = x.view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def _np(t):
    if t is None:
        return None
    if hasattr(t, "detach"):
        t = t.detach().double().numpy()
    return np.asarray(t, dtype=np.float64)


def frame_solve(K, V, beta, G, block, diag_inverse=False, rnd=lambda x: x):
    """Blocked forward substitution of (I + A)[Ub | W] = R.  With
    ``diag_inverse`` each diagonal block is applied through its explicit
    inverse (as a tensor-core kernel would); ``rnd`` models operand rounding."""
    L = K.shape[0]
    R = np.concatenate([beta[:, None] * V, (beta * np.exp(G))[:, None] * K], axis=1)
    X = np.zeros_like(R)
    for r0 in range(0, L, block):
        r1 = min(r0 + block, L)
        acc = R[r0:r1].copy()
        for s0 in range(0, r0, block):
            s1 = s0 + block
            A = beta[r0:r1, None] * (K[r0:r1] @ K[s0:s1].T) * np.exp(G[r0:r1, None] - G[None, s0:s1])
            acc -= rnd(A) @ rnd(X[s0:s1])
        Ad = np.tril(beta[r0:r1, None] * (K[r0:r1] @ K[r0:r1].T) * np.exp(G[r0:r1, None] - G[None, r0:r1]), -1)
        if diag_inverse:
            Tinv = np.linalg.inv(np.eye(r1 - r0) + Ad)
            X[r0:r1] = rnd(Tinv) @ rnd(acc)
        else:
            for i in range(r1 - r0):
                acc[i] -= Ad[i, :i] @ acc[:i]
            X[r0:r1] = acc
    return X


def chunk_forward(q, k, v, alpha, beta, S_in, frame_len, block=32, diag_inverse=False, bf16=False):
    q, k, v, alpha, beta, S_in = (_np(t) for t in (q, k, v, alpha, beta, S_in))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    rnd = _bf16 if bf16 else (lambda x: x)
    o = np.zeros((B, T, H, dv))
    S_out = np.zeros((B, H, dv, dk))
    L = frame_len
    for b in range(B):
        for h in range(H):
            Sig = np.zeros((dk, dv)) if S_in is None else S_in[b, h].T.copy()
            for f in range(T // L):
                sl = slice(f * L, (f + 1) * L)
                Q, K, V = q[b, sl, h], k[b, sl, h], v[b, sl, h]
                la = np.maximum(np.log(np.maximum(alpha[b, sl, h], 1e-300)), LOG_FLOOR)
                G = np.cumsum(la)
                bt = beta[b, sl, h]
                X = frame_solve(K, V, bt, G, block, diag_inverse, rnd)
                Ub, Wm = X[:, :dv], X[:, dv:]
                U = Ub - rnd(Wm) @ rnd(Sig)
                Kt = np.exp(G[-1] - G)[:, None] * K
                M = np.exp(G[-1]) * np.eye(dk) - rnd(Kt).T @ rnd(Wm)
                N = rnd(Kt).T @ rnd(Ub)
                P = np.tril((Q @ K.T) * np.exp(np.minimum(G[:, None] - G[None, :], 0.0)))
                o[b, sl, h] = np.exp(G)[:, None] * (rnd(Q) @ rnd(Sig)) + rnd(P) @ rnd(U)
                Sig = M @ Sig + N
            S_out[b, h] = Sig.T
    return o, S_out
