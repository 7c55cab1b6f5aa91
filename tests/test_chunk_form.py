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
