"""fp64 numpy restatement of the chunkwise form of the gated delta rule.

Test-only.  It states the algebra the CUDA kernels are built on, so that the
derivation itself is checked against the token-loop oracle before any kernel
is trusted; the CUDA path shares no code with it.

Sources: "Hybrid Linear Attention Architecture Design Explained", section 4
(cross-chunk state update and intra-chunk output with cumulative decay, a
lower-triangular mask and the correction U - W S), written here in the
d_v x d_k state convention of "From Traditional Attention to hybrid ones"
(section 5); "Hybrid attention", "Training a recurrence in parallel" (the
intra-chunk dependencies are a lower-triangular system; only the state passes
between chunks).

Within one chunk of C tokens with start state S0 (d_v x d_k), b_i = sum_{j<=i} g_j
(a vector over d_k for the per-channel gate), Gam_i = exp(b_i):
  A  = strictly-lower part of diag(beta) (K*Gam) (K/Gam)^T
  W  = (I + A)^-1 diag(beta) (K*Gam)        U = (I + A)^-1 diag(beta) V
  U' = U - W S0^T                            (the delta-corrected writes)
  O  = (Q*Gam) S0^T + tril_incl((Q*Gam)(K/Gam)^T) U'
  S  = S0 Diag(Gam_C) + U'^T (K * Gam_C/Gam)
"""
import numpy as np


def chunk_forward(q, k, v, g, beta, S0=None, C=64, scale=1.0):
    """One sequence, one head: q,k (T,dk), v (T,dv), g (T,) or (T,dk), beta (T,)."""
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else S0.astype(np.float64).copy()
    out = np.zeros((T, dv))
    for s in range(0, T, C):
        e = min(T, s + C)
        Q, K, V, be = q[s:e] * scale, k[s:e], v[s:e], beta[s:e]
        gg = g[s:e] if g.ndim == 2 else g[s:e][:, None] * np.ones((1, dk))
        b = np.cumsum(gg, axis=0)
        Gam = np.exp(b)
        Kd, Ki = K * Gam, K / Gam
        n = e - s
        A = np.tril(be[:, None] * (Kd @ Ki.T), -1)
        Tinv = np.linalg.solve(np.eye(n) + A, np.eye(n))
        W = Tinv @ (be[:, None] * Kd)
        U = Tinv @ (be[:, None] * V)
        Up = U - W @ S.T
        out[s:e] = (Q * Gam) @ S.T + np.tril((Q * Gam) @ Ki.T) @ Up
        S = S * Gam[-1][None, :] + Up.T @ (K * (Gam[-1][None, :] / Gam))
    return out, S
