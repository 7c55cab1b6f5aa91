"""fp64 CPU oracle of the work before the gated delta rule -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may use
it; the CUDA library never does.

What a Gated DeltaNet layer does to its projections before the recurrence
("Attention, Part 4: Linear Attention, Gated DeltaNet and Hybrid Models",
section 6, "Where alpha and beta come from", and the paragraph after it;
"From Traditional Attention to hybrid ones", sections 6 and "vLLM Storage" for
the convolution history kept per live sequence):

  * the query, key and value channels of each token pass through a short causal
    depthwise convolution over the last K tokens, then SiLU;
  * queries and keys are then normalised to length 1 per head;
  * beta = sigmoid(b);
  * g = log(alpha) = -exp(A_log) * softplus(a + dt_bias), per value head.

Readings where the pages are silent (stated in the design notes as well):
  * the convolution and SiLU apply to q, k and v alike (the pages name the q/k
    path; the value channels are part of the same mixed projection), the L2 norm
    to q and k only;
  * tap j of a channel's K weights multiplies the input K-1-j tokens back (the
    last tap the current token); there is no bias;
  * the length-1 normalisation is x / sqrt(sum x^2 + 1e-6), so that an all-zero
    head stays finite;
  * the convolution history of a sequence is its last K-1 raw inputs, oldest
    first; positions before a sequence's first token read that history (zeros
    when none is given).

Everything is plain numpy in float64, one token at a time.
"""
from __future__ import annotations

import numpy as np

L2_EPS = 1e-6


def _f64(t):
    if t is None:
        return None
    if hasattr(t, "detach"):
        t = t.detach().cpu()
        if str(t.dtype) == "torch.bfloat16":
            t = t.float()
        t = t.double().numpy()
    return np.asarray(t, dtype=np.float64)


def silu(x):
    return x / (1.0 + np.exp(-x))


def sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def softplus(x):
    # log(1 + e^x) without overflow
    return np.where(x > 30.0, x, np.log1p(np.exp(np.minimum(x, 30.0))))


def prerule(x, a, b, conv_w, A_log, dt_bias, *, hk, dk, H, dv, cu_seqlens=None, conv_state=None):
    """x: (B, T, C) with C = 2 hk dk + H dv, channels [q heads | k heads | v heads];
    a, b: (B, T, H); conv_w: (C, K); A_log, dt_bias: (H,); cu_seqlens: None (B
    sequences of T tokens) or N+1 offsets into the B*T rows; conv_state: (N, C, K-1)
    or None.  Returns q (B,T,hk,dk), k (B,T,hk,dk), v (B,T,H,dv), g (B,T,H),
    beta (B,T,H) and the new convolution history (N, C, K-1), all float64."""
    x, a, b, w = _f64(x), _f64(a), _f64(b), _f64(conv_w)
    A_log, dt_bias, hist = _f64(A_log), _f64(dt_bias), _f64(conv_state)
    B, T, C = x.shape
    K = w.shape[1]
    assert C == 2 * hk * dk + H * dv and w.shape[0] == C
    rows = x.reshape(B * T, C)
    if cu_seqlens is None:
        starts = [n * T for n in range(B)]
        lens = [T] * B
    else:
        cs = [int(c) for c in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
        starts, lens = cs[:-1], [cs[i + 1] - cs[i] for i in range(len(cs) - 1)]
    N = len(starts)
    y = np.zeros((B * T, C))
    new_hist = np.zeros((N, C, K - 1))
    for n in range(N):
        s, L = starts[n], lens[n]
        past = np.zeros((C, K - 1)) if hist is None else hist[n]

        def inp(p):  # raw input at position p of sequence n (p may be negative)
            return rows[s + p] if p >= 0 else past[:, K - 1 + p]

        for p in range(L):
            acc = np.zeros(C)
            for j in range(K):
                acc += w[:, j] * inp(p - (K - 1) + j)
            y[s + p] = silu(acc)
        for j in range(K - 1):
            new_hist[n, :, j] = inp(L - (K - 1) + j)
    y = y.reshape(B, T, C)
    q = y[..., : hk * dk].reshape(B, T, hk, dk)
    k = y[..., hk * dk: 2 * hk * dk].reshape(B, T, hk, dk)
    v = y[..., 2 * hk * dk:].reshape(B, T, H, dv)
    q = q / np.sqrt(np.sum(q * q, axis=-1, keepdims=True) + L2_EPS)
    k = k / np.sqrt(np.sum(k * k, axis=-1, keepdims=True) + L2_EPS)
    beta = sigmoid(b)
    g = -np.exp(A_log) * softplus(a + dt_bias)
    return q, k, v, g, beta, new_hist
