"""Pins of the pre-rule oracle (CPU only): the short causal convolution, SiLU, the
q/k normalisation and the gates, each checked against something other than the
oracle's own formula -- a library convolution, closed-form gate values,
invariants (causality, continuation through the convolution history, packing) --
and a few planted mistakes that must fail at least one pin."""
import inspect
import math
import types

import numpy as np
import pytest

from oracle import prerule as P


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _setup(seed=0, B=2, T=9, hk=1, dk=4, H=2, dv=4, K=4):
    rng = np.random.default_rng(seed)
    C = 2 * hk * dk + H * dv
    return dict(x=_rand(rng, B, T, C), a=_rand(rng, B, T, H), b=_rand(rng, B, T, H), conv_w=_rand(rng, C, K),
                A_log=_rand(rng, H) * 0.5, dt_bias=_rand(rng, H) * 0.5, hk=hk, dk=dk, H=H, dv=dv)


def _v_channels(kw):
    return 2 * kw["hk"] * kw["dk"]


# ---------------------------------------------------------------------------
# pins
# ---------------------------------------------------------------------------

def pin_matches_library_convolution(mod):
    """Value channels (SiLU only) equal SiLU of numpy's full convolution with the
    taps reversed, truncated (the layer's convolution is a cross-correlation: its
    last tap multiplies the current token): fixes the orientation of the taps and
    the causal alignment."""
    kw = _setup(1)
    q, k, v, g, beta, _ = mod.prerule(**kw)
    x, w = kw["x"], kw["conv_w"]
    c0 = _v_channels(kw)
    B, T, _ = x.shape
    for bb in range(B):
        for c in range(kw["H"] * kw["dv"]):
            ref = np.convolve(x[bb, :, c0 + c], w[c0 + c][::-1])[:T]
            got = v[bb, :, c // kw["dv"], c % kw["dv"]]
            assert np.allclose(got, ref / (1 + np.exp(-ref)), rtol=0, atol=1e-13)


def pin_impulse_response(mod):
    """A unit impulse on one value channel reads back its K weights, newest tap first."""
    kw = _setup(2, B=1, T=8)
    kw["x"] = np.zeros_like(kw["x"])
    c0, K = _v_channels(kw), kw["conv_w"].shape[1]
    kw["x"][0, 3, c0 + 1] = 1.0
    _, _, v, _, _, _ = mod.prerule(**kw)
    col = v[0, :, 0, 1]
    w = kw["conv_w"][c0 + 1]
    for t in range(8):
        m = t - 3
        expect = w[K - 1 - m] if 0 <= m < K else 0.0
        assert math.isclose(col[t], expect / (1 + math.exp(-expect)), abs_tol=1e-15)


def pin_causal(mod):
    kw = _setup(3)
    base = mod.prerule(**kw)
    kw["x"] = kw["x"].copy()
    kw["x"][:, 6:] += 5.0
    moved = mod.prerule(**kw)
    for a, b in zip(base[:3], moved[:3]):
        assert np.array_equal(a[:, :6], b[:, :6])


def pin_history_continuation(mod):
    """Two calls with the history carried equal one call (fp64, exactly)."""
    kw = _setup(4, B=1, T=11)
    full = mod.prerule(**kw)
    part = lambda s, e: {**kw, "x": kw["x"][:, s:e], "a": kw["a"][:, s:e], "b": kw["b"][:, s:e]}
    first = mod.prerule(**part(0, 5))
    second = mod.prerule(**part(5, 11), conv_state=first[5])
    for i in range(5):
        assert np.array_equal(np.concatenate([first[i], second[i]], axis=1), full[i])
    assert np.array_equal(second[5], full[5])
    # a sequence shorter than the history keeps the older part of it
    third = mod.prerule(**part(5, 6), conv_state=first[5])
    K = kw["conv_w"].shape[1]
    assert np.array_equal(third[5][:, :, : K - 2], first[5][:, :, 1:])
    assert np.array_equal(third[5][0, :, K - 2], kw["x"][0, 5])


def pin_packing(mod):
    """Packed sequences equal separate runs; no convolution reads across a boundary."""
    kw = _setup(5, B=1, T=12)
    cu = [0, 3, 3, 10, 12]
    packed = mod.prerule(**kw, cu_seqlens=cu)
    for n in range(4):
        s, e = cu[n], cu[n + 1]
        if e == s:
            assert np.array_equal(packed[5][n], np.zeros_like(packed[5][n]))
            continue
        one = mod.prerule(**{**kw, "x": kw["x"][:, s:e], "a": kw["a"][:, s:e], "b": kw["b"][:, s:e]})
        for i in range(5):
            assert np.array_equal(packed[i][:, s:e], one[i])
        assert np.array_equal(packed[5][n], one[5][0])


def pin_unit_length_queries(mod):
    """q and k heads are the value path's vectors scaled to length 1: feeding the same
    raw channels and weights to a query head, a key head and a value head
    (d_k = d_v) gives q = k = v / sqrt(|v|^2 + eps)."""
    kw = _setup(6, B=1, T=7, hk=1, dk=4, H=1, dv=4)
    x, w = kw["x"], kw["conv_w"]
    x[..., 0:4] = x[..., 8:12]
    x[..., 4:8] = x[..., 8:12]
    w[0:4] = w[8:12]
    w[4:8] = w[8:12]
    q, k, v, _, _, _ = mod.prerule(**kw)
    vv = v[0, :, 0]
    n2 = np.sum(vv * vv, axis=-1, keepdims=True)
    for t in (q, k):
        assert np.allclose(t[0, :, 0], vv / np.sqrt(n2 + 1e-6), rtol=1e-14, atol=0)
        assert np.all(np.abs(np.sum(t[0, :, 0] ** 2, axis=-1) - 1) < 1e-5)


def pin_gate_values(mod):
    """Closed forms.  Head 0 (A_log = dt_bias = 0): a = 0 gives g = -ln 2, and
    softplus(1) - softplus(-1) = 1.  Head 1 (A_log = ln 2, dt_bias = ln(e - 1), so
    softplus(0 + dt_bias) = 1): a = 0 gives g = -2 exactly; g -> 0- as a -> -inf and
    g -> -2 (a + dt_bias) for large a.  beta(0) = 1/2, beta(b) + beta(-b) = 1; g < 0."""
    kw = _setup(7, B=1, T=5, H=2)
    kw["a"] = np.array([[[0.0, 0.0], [0.0, -60.0], [1.0, 40.0], [-1.0, 0.0], [0.0, 0.0]]])
    kw["b"] = np.array([[[0.0, 3.0], [-3.0, 0.0], [0.0, 0.0], [0.0, 0.0], [0.0, 0.0]]])
    kw["A_log"] = np.array([0.0, math.log(2.0)])
    kw["dt_bias"] = np.array([0.0, math.log(math.e - 1.0)])
    _, _, _, g, beta, _ = mod.prerule(**kw)
    assert math.isclose(g[0, 0, 0], -math.log(2.0), rel_tol=1e-15)
    assert math.isclose(g[0, 2, 0] - g[0, 3, 0], -1.0, rel_tol=1e-14)
    assert math.isclose(g[0, 0, 1], -2.0, rel_tol=1e-14)
    assert -1e-25 < g[0, 1, 1] < 0
    assert math.isclose(g[0, 2, 1], -2.0 * (40.0 + math.log(math.e - 1.0)), rel_tol=1e-14)
    assert math.isclose(beta[0, 0, 0], 0.5, rel_tol=0, abs_tol=0)
    assert math.isclose(beta[0, 0, 1] + beta[0, 1, 0], 1.0, rel_tol=1e-15)
    assert np.all(g < 0) and np.all((beta > 0) & (beta < 1))


PINS = [pin_matches_library_convolution, pin_impulse_response, pin_causal, pin_history_continuation, pin_packing,
        pin_unit_length_queries, pin_gate_values]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(P)


# ---------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# ---------------------------------------------------------------------------

MUTANTS = {
    "taps reversed": ("acc += w[:, j] * inp(p - (K - 1) + j)", "acc += w[:, K - 1 - j] * inp(p - (K - 1) + j)"),
    "window shifted": ("acc += w[:, j] * inp(p - (K - 1) + j)", "acc += w[:, j] * inp(p - K + j)"),
    "history newest first": ("return rows[s + p] if p >= 0 else past[:, K - 1 + p]",
                             "return rows[s + p] if p >= 0 else past[:, -1 - (K - 1 + p)]"),
    "no SiLU": ("y[s + p] = silu(acc)", "y[s + p] = acc"),
    "norm epsilon": ("np.sum(q * q, axis=-1, keepdims=True) + L2_EPS", "np.sum(q * q, axis=-1, keepdims=True) + 1.0"),
    "gate sign": ("g = -np.exp(A_log) * softplus(a + dt_bias)", "g = np.exp(A_log) * softplus(a + dt_bias)"),
    "bias outside": ("g = -np.exp(A_log) * softplus(a + dt_bias)", "g = -np.exp(A_log) * (softplus(a) + dt_bias)"),
    "history not carried": ("past = np.zeros((C, K - 1)) if hist is None else hist[n]", "past = np.zeros((C, K - 1))"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    old, new = MUTANTS[name]
    src = inspect.getsource(P)
    assert old in src, name
    mod = types.ModuleType("prerule_mutant")
    exec(compile(src.replace(old, new), "prerule_mutant", "exec"), mod.__dict__)
    failed = 0
    for pin in PINS:
        try:
            pin(mod)
        except Exception:
            failed += 1
    assert failed > 0, f"no pin catches: {name}"
