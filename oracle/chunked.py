"""numpy fp64 chunked closed form of the gated delta rule -- TEST INFRASTRUCTURE ONLY.

Used only to cross-check the token-by-token oracle (``oracle.forward``) on small
inputs; it is a second, independent formulation of the same layer, not a model of
the GPU kernels (it shares nothing with them).

Derivation, for one sequence and one V head (state S is d_v x d_k, rows of Q, K, V
are tokens).  Writing the update as S_t = a_t S_{t-1} + d_t k_t^T with
d_t = b_t (v_t - a_t S_{t-1} k_t), and unrolling over a chunk that enters with state
S0 and has in-chunk inclusive gate sums G_r = g_1 + ... + g_r:

  * A[r, j] = b_r exp(G_r - G_j) (k_r . k_j) for j < r (else 0), so that the chunk's
    corrections Delta (rows d_r) satisfy (I + A) Delta = diag(b) V - diag(b gamma) K S0^T,
    with gamma_r = exp(G_r);
  * T = (I + A)^-1, W = T diag(b gamma) K, U = T diag(b) V, Delta = U - W S0^T;
  * P[r, j] = exp(G_r - G_j) (q_r . k_j) for j <= r (else 0);
    outputs O = diag(gamma) Q S0^T + P Delta;
  * the state leaving the chunk is gamma_last S0 + Delta^T diag(c) K with
    c_j = exp(G_last - G_j).

Decays are always formed as exp(G_r - G_j) with r >= j, never as a ratio of
cumulative products.
"""

from __future__ import annotations

import numpy as np


def normalise(q, k, eps):
    """Row-wise L2 normalisation; q is also scaled by 1/sqrt(d_k)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    dk = q.shape[-1]
    qn = q / np.sqrt((q * q).sum(-1, keepdims=True) + eps) / np.sqrt(dk)
    kn = k / np.sqrt((k * k).sum(-1, keepdims=True) + eps)
    return qn, kn


def chunk_step(Qn, Kn, V, g, b, S0):
    """One chunk of the closed form. Returns (O [L, dv], S_out [dv, dk])."""
    L = Qn.shape[0]
    G = np.cumsum(g)
    gamma = np.exp(G)
    r = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    diff = np.where(r >= j, G[:, None] - G[None, :], -np.inf)
    decay = np.exp(diff)                        # exp(G_r - G_j) on and below the diagonal
    A = np.where(r > j, b[:, None] * decay * (Kn @ Kn.T), 0.0)
    P = np.where(r >= j, decay * (Qn @ Kn.T), 0.0)
    IA = np.eye(L) + A
    W = np.linalg.solve(IA, (b * gamma)[:, None] * Kn)
    U = np.linalg.solve(IA, b[:, None] * V)
    Delta = U - W @ S0.T
    O = gamma[:, None] * (Qn @ S0.T) + P @ Delta
    c = np.exp(G[-1] - G)
    S_out = gamma[-1] * S0 + Delta.T @ (c[:, None] * Kn)
    return O, S_out


def chunked_forward(q, k, v, g, beta, S0=None, chunk=64, eps=1e-6):
    """Chunked closed form for ONE sequence and ONE V head.

    q, k: [T, dk] (raw, normalised here); v: [T, dv]; g, beta: [T]; S0: [dv, dk] or None.
    Returns (out [T, dv], S_T [dv, dk]).
    """
    Qn, Kn = normalise(q, k, eps)
    V = np.asarray(v, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    b = np.asarray(beta, dtype=np.float64)
    T, dk = Qn.shape
    dv = V.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    out = np.zeros((T, dv))
    for c0 in range(0, T, chunk):
        c1 = min(c0 + chunk, T)
        O, S = chunk_step(Qn[c0:c1], Kn[c0:c1], V[c0:c1], g[c0:c1], b[c0:c1], S)
        out[c0:c1] = O
    return out, S
