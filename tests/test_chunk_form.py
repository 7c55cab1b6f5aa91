"""The chunk algebra the kernels implement equals the token-loop oracle (CPU).

"Hybrid attention" ("Training a recurrence in parallel") reports the chunked
form agreeing with the token loop to 1.4e-15 in double precision; the bound
here is 1e-12 relative to the output scale.
"""
import numpy as np
import pytest

import oracle
from tests.chunk_form import chunk_forward


def _problem(seed, T, dk, dv, per_channel, gate_mu=-2.0):
    r = np.random.default_rng(seed)
    unit = lambda a: a / np.linalg.norm(a, axis=-1, keepdims=True)
    q, k = unit(r.standard_normal((T, dk))), unit(r.standard_normal((T, dk)))
    v = r.standard_normal((T, dv))
    beta = 1 / (1 + np.exp(-r.standard_normal(T)))
    x = r.standard_normal((T, dk) if per_channel else T) + gate_mu
    g = -np.logaddexp(0, x)
    S0 = r.standard_normal((dv, dk)) * 0.3
    return q, k, v, g, beta, S0


@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("C,T", [(16, 100), (64, 200), (64, 64), (64, 5)])
def test_chunk_form_matches_token_loop(per_channel, C, T):
    q, k, v, g, beta, S0 = _problem(C * 1000 + T, T, 12, 9, per_channel)
    o_ref, s_ref, _ = oracle.gated_delta_rule(q[None, :, None], k[None, :, None], v[None, :, None],
                                              g[None, :, None], beta[None, :, None], S0[None, None],
                                              per_channel=per_channel, scale=0.7)
    o, s = chunk_forward(q, k, v, g, beta, S0, C=C, scale=0.7)
    assert np.max(np.abs(o - o_ref[0, :, 0])) <= 1e-12 * max(1, np.abs(o_ref).max())
    assert np.max(np.abs(s - s_ref[0, 0])) <= 1e-12 * max(1, np.abs(s_ref).max())


def test_chunk_form_long_memory_gates():
    """alpha close to 1 (gate x ~ N(-7, 1)) so that the state carries across many chunks."""
    q, k, v, g, beta, S0 = _problem(7, 300, 16, 8, False, gate_mu=-7.0)
    o_ref, s_ref, _ = oracle.gated_delta_rule(q[None, :, None], k[None, :, None], v[None, :, None],
                                              g[None, :, None], beta[None, :, None], S0[None, None])
    o, s = chunk_forward(q, k, v, g, beta, S0, C=64)
    assert np.max(np.abs(o - o_ref[0, :, 0])) <= 1e-12 * max(1, np.abs(o_ref).max())
    assert np.max(np.abs(s - s_ref[0, 0])) <= 1e-12 * max(1, np.abs(s_ref).max())


@pytest.mark.parametrize("per_channel", [False, True])
def test_segment_end_state_is_affine_in_its_start(per_channel):
    """The sequence split rests on this: over a run of chunks the end state is
    S_end = S_start M + B, with B the end state from a zero start and M the end state
    from the identity start with the writes dropped (v = 0; d_v = d_k)."""
    d = 10
    q, k, v, g, beta, _ = _problem(31, 230, d, d, per_channel)
    X = np.random.default_rng(32).standard_normal((d, d))
    _, S_x = chunk_forward(q, k, v, g, beta, X, C=64)
    _, B = chunk_forward(q, k, v, g, beta, np.zeros((d, d)), C=64)
    _, M = chunk_forward(q, k, np.zeros_like(v), g, beta, np.eye(d), C=64)
    assert np.max(np.abs(S_x - (X @ M + B))) <= 1e-12 * max(1, np.abs(S_x).max())


def test_one_group_form_of_a_chunk():
    """Substituting U' = U - W S0^T, one product [S0 | U^T] [[-W^T K~, -W^T P^T, Qs^T],
    [K~, P^T, 0]] gives the state increment S - gam_L S0 and the output in two parts
    (the one-MMA-group form of a chunk, worked out as an alternative to the two groups)."""
    C, dk, dv = 64, 12, 9
    q, k, v, g, beta, S0 = _problem(34, C, dk, dv, False)
    o_ref, s_ref = chunk_forward(q, k, v, g, beta, S0, C=C)
    b = np.cumsum(g)
    Gam = np.exp(b)
    Kd, Ki = k * Gam[:, None], k / Gam[:, None]
    A = np.tril(beta[:, None] * (Kd @ Ki.T), -1)
    Tinv = np.linalg.inv(np.eye(C) + A)
    W, U = Tinv @ (beta[:, None] * Kd), Tinv @ (beta[:, None] * v)
    Qs = q * Gam[:, None]
    P = np.tril(Qs @ Ki.T)
    Kt = k * np.exp(b[-1] - b)[:, None]
    top = np.hstack([-W.T @ Kt, -W.T @ P.T, Qs.T])           # d_k x (d_k + 2 C)
    bottom = np.hstack([Kt, P.T, np.zeros((C, C))])         # C x (d_k + 2 C)
    D = np.hstack([S0, U.T]) @ np.vstack([top, bottom])      # d_v x (d_k + 2 C)
    s = Gam[-1] * S0 + D[:, :dk]
    o = (D[:, dk:dk + C] + D[:, dk + C:]).T
    assert np.max(np.abs(s - s_ref)) <= 1e-12 * max(1, np.abs(s_ref).max())
    assert np.max(np.abs(o - o_ref)) <= 1e-12 * max(1, np.abs(o_ref).max())


def _grouped_forward(q, k, v, g, beta, S0, C=64, scale=1.0):
    """The chunk step regrouped the way the tensor-core kernels form it, chunk by chunk:
    the block holds W^T = (T diag(beta gam) K)^T (per-channel gate: T diag(beta) (K*Gam)),
    P and -T'' = -T diag(beta), never U; the scan's first group gives
    D = S0 W^T + V^T (-T'')^T = -U'^T, so U' = -D^T; the state increment is
    (diag(w) U')^T K with w_j = exp(b_L - b_j) for one gate per head (U'^T K~ with
    K~ = K * exp(b_L - b) per channel); the output is scale gam_i (S0 q_i) + P U'."""
    T, dk = k.shape
    per_channel = g.ndim == 2
    S = S0.astype(np.float64).copy()
    out = np.zeros((T, v.shape[1]))
    for s0 in range(0, T, C):
        e = min(T, s0 + C)
        n = e - s0
        Q, K, V, be = q[s0:e], k[s0:e], v[s0:e], beta[s0:e]
        b = np.cumsum(g[s0:e], axis=0)
        dec = np.exp(b[:, None, :] - b[None, :, :]) if per_channel else np.exp(b[:, None] - b[None, :])
        gram = np.einsum("ic,jc,ijc->ij", K, K, dec) if per_channel else (K @ K.T) * dec
        qk = np.einsum("ic,jc,ijc->ij", Q, K, dec) if per_channel else (Q @ K.T) * dec
        Tm = np.linalg.inv(np.eye(n) + np.tril(be[:, None] * gram, -1))
        Tb = Tm * be[None, :]                                  # T'' = T diag(beta)
        Wt = (Tb @ (K * np.exp(b))).T if per_channel else (Tm * (be * np.exp(b))[None, :] @ K).T
        P = scale * np.tril(qk)
        D = S @ Wt + V.T @ (-Tb).T                              # -U'^T
        Up = -D.T
        if per_channel:
            inc = Up.T @ (K * np.exp(b[-1] - b))
            out[s0:e] = (scale * Q * np.exp(b)) @ S.T + P @ Up
            S = S * np.exp(b[-1])[None, :] + inc
        else:
            w = np.exp(b[-1] - b)
            inc = (w[:, None] * Up).T @ K
            out[s0:e] = (scale * np.exp(b))[:, None] * (Q @ S.T) + P @ Up
            S = np.exp(b[-1]) * S + inc
    return out, S


@pytest.mark.parametrize("per_channel", [False, True])
def test_kernel_grouping_matches_token_loop(per_channel):
    """The regrouping the kernels use (no U in the block; -U'^T as one accumulation of
    S0 W^T and V^T (-T'')^T; the increment through diag(w) U' for one gate per head)
    is the same chunk step: equal to the token loop over several chunks and a ragged
    tail."""
    q, k, v, g, beta, S0 = _problem(41, 150, 12, 9, per_channel)
    o_ref, s_ref, _ = oracle.gated_delta_rule(q[None, :, None], k[None, :, None], v[None, :, None],
                                              g[None, :, None], beta[None, :, None], S0[None, None],
                                              per_channel=per_channel, scale=0.7)
    o, s = _grouped_forward(q, k, v, g, beta, S0, C=64, scale=0.7)
    assert np.max(np.abs(o - o_ref[0, :, 0])) <= 1e-12 * max(1, np.abs(o_ref).max())
    assert np.max(np.abs(s - s_ref[0, 0])) <= 1e-12 * max(1, np.abs(s_ref).max())


@pytest.mark.parametrize("L", [64, 40, 17])
def test_per_channel_blocks_as_one_product(L):
    """The per-channel prep forms A and P as one product when the decays are
    moderate: with m = b at row 31 (b constant after row L - 1), E+_i = exp(b_i - m),
    E-_j = exp(m - b_j), beta_i (K*E+)(K*E-)^T below the diagonal is A and
    (Q*E+)(K*E-)^T on and below it is P; the entries above are dropped by selection."""
    dk = 16
    q, k, _, g, beta, _ = _problem(36 + L, 64, dk, 4, True, gate_mu=0.5)
    g[L:] = 0.0
    beta[L:] = 0.0
    b = np.cumsum(g, axis=0)
    dec = np.exp(b[:, None, :] - b[None, :, :])               # exp(b_i - b_j) per channel
    A_def = np.tril(beta[:, None] * np.einsum("ic,jc,ijc->ij", k, k, dec), -1)
    P_def = np.tril(np.einsum("ic,jc,ijc->ij", q, k, dec))
    m = b[31]
    Ep, Em = np.exp(b - m), np.exp(m - b)
    full_a = beta[:, None] * ((k * Ep) @ (k * Em).T)
    full_p = (q * Ep) @ (k * Em).T
    i, j = np.indices((64, 64))
    A = np.where((j < i) & (i < L), full_a, 0.0)
    P = np.where((j <= i) & (i < L), full_p, 0.0)
    P_def[L:] = 0.0
    assert np.max(np.abs(A - A_def)) <= 1e-12 * max(1, np.abs(A_def).max())
    assert np.max(np.abs(P - P_def)) <= 1e-12 * max(1, np.abs(P_def).max())


@pytest.mark.parametrize("per_channel", [False, True])
def test_decay_bound_of_a_chunk(per_channel):
    """The split scan drops a segment's start state once the summed decay bound of the
    chunks before falls below 2^-126.  The bound: with 0 <= beta_t |k_t|^2 <= 2 every
    factor (I - beta_t k_t k_t^T) is a contraction, so the homogeneous map of a run
    of tokens (the writes dropped) has spectral norm <= prod_t max_c alpha_{t,c}; the
    kernels store log2 of that product per chunk.  Checked in fp64 on runs of 64
    tokens with keys of length up to sqrt(2) and beta up to 1, and with beta = 1."""
    d = 16
    r = np.random.default_rng(33)
    for trial in range(20):
        q, k, v, g, beta, _ = _problem(40 + trial, 64, d, d, per_channel, gate_mu=-5.0)
        k = k * r.uniform(0.2, np.sqrt(2.0), size=(64, 1))  # |k|^2 up to 2 with beta <= 1
        if trial % 2:
            beta = np.ones_like(beta)
            k = k / np.linalg.norm(k, axis=1, keepdims=True)
        _, M = chunk_forward(q, k, np.zeros_like(v), g, beta, np.eye(d), C=64)  # the map S0 -> S0 M
        gmax = g if g.ndim == 1 else g.max(axis=1)
        bound = np.exp(gmax.sum())
        assert np.linalg.norm(M, 2) <= bound * (1 + 1e-12), (np.linalg.norm(M, 2), bound)


def test_zero_start_outputs_after_the_bound_match():
    """A run whose summed decay bound falls below 2^-126: from there on its outputs and
    state from a zero start equal those from the true start to far below fp32
    resolution (the split scan takes them from the zero-start pass)."""
    q, k, v, g, beta, S0 = _problem(51, 640, 16, 16, False, gate_mu=1.0)  # strong decay
    lam = np.cumsum(g) / np.log(2.0)
    m = int(np.argmax(lam < -126.0))
    assert 0 < m < 600
    o_true, s_true = chunk_forward(q, k, v, g, beta, S0 * 100.0, C=64)
    o_zero, s_zero = chunk_forward(q, k, v, g, beta, np.zeros_like(S0), C=64)
    scale = np.abs(o_true).max()
    assert np.max(np.abs(o_true[m + 1:] - o_zero[m + 1:])) <= 2.0 ** -100 * scale
    assert np.max(np.abs(s_true - s_zero)) <= 2.0 ** -100 * max(1.0, np.abs(s_true).max())
