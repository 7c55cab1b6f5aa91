"""GPU parity of gdn_prerule (the work before the recurrence) against the fp64
pre-rule oracle on the same seeded raw projections, and the whole layer core
(pre-rule then chunked prefill) against the two oracles chained."""
import numpy as np
import pytest
import torch

import oracle
from oracle import prerule as P
from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import make_prerule_inputs
from tests.gpu_util import rel_l2

pytestmark = pytest.mark.gpu


def _run(pi, *, hist_out=True, alias=False):
    d = lambda t: None if t is None else t.cuda().contiguous()
    hist_in = d(pi.hist)
    out_hist = None
    if hist_out:
        N = (pi.cu_seqlens.numel() - 1) if pi.cu_seqlens is not None else pi.x.shape[0]
        out_hist = hist_in if (alias and hist_in is not None) else torch.full(
            (N, pi.x.shape[-1], pi.conv_w.shape[1] - 1), float("nan"), device="cuda")
    res = gdn.gdn_prerule(d(pi.x), d(pi.a), d(pi.b), d(pi.conv_w), d(pi.A_log), d(pi.dt_bias), hk=pi.hk, dk=pi.dk,
                          H=pi.H, dv=pi.dv, cu_seqlens=d(pi.cu_seqlens), conv_state_in=hist_in,
                          conv_state_out=out_hist)
    torch.cuda.synchronize()
    return res, out_hist


def _oracle(pi):
    return P.prerule(pi.x, pi.a, pi.b, pi.conv_w, pi.A_log, pi.dt_bias, hk=pi.hk, dk=pi.dk, H=pi.H, dv=pi.dv,
                     cu_seqlens=pi.cu_seqlens, conv_state=pi.hist)


def _check(pi, res, hist, ref, rows=None):
    tol = 1e-5 if pi.x.dtype == torch.float32 else 1e-2
    names = ("q", "k", "v", "log_gate", "beta")
    for name, got, want in zip(names, res, ref[:5]):
        g_, w_ = got.cpu().double().numpy(), want
        if rows is not None:
            g_, w_ = g_.reshape(-1, *g_.shape[2:])[rows], w_.reshape(-1, *w_.shape[2:])[rows]
        t = 1e-5 if name in ("log_gate", "beta") else tol
        assert rel_l2(g_, w_) <= t, name
    if hist is not None:
        assert np.array_equal(hist.cpu().double().numpy(), ref[5])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("K", [4, 2])
def test_fixed_length(dtype, d, K):
    pi = make_prerule_inputs(B=3, T=37, H=4, hk=2, dk=d, dv=d, K=K, dtype=dtype, seed=50 + K)
    res, hist = _run(pi)
    _check(pi, res, hist, _oracle(pi))


def test_no_history_and_in_place_history():
    pi = make_prerule_inputs(B=2, T=20, H=2, hk=2, dk=128, dv=128, dtype="bf16", history=False, seed=54)
    res, hist = _run(pi)
    _check(pi, res, hist, _oracle(pi))
    pi = make_prerule_inputs(B=2, T=2, H=2, hk=1, dk=128, dv=128, dtype="bf16", seed=55)  # T < K - 1
    ref = _oracle(pi)
    res, hist = _run(pi, alias=True)
    _check(pi, res, hist, ref)


def test_packed():
    lengths = [5, 0, 1, 40, 2, 17]
    pi = make_prerule_inputs(B=1, T=0, H=4, hk=4, dk=64, dv=128, dtype="bf16", lengths=lengths, seed=56)
    res, hist = _run(pi)
    _check(pi, res, hist, _oracle(pi))


def test_decode_steps_continue_prefill():
    """Prefill of 30 tokens then 6 single-token steps (history in place) equal one
    pass over all 36 tokens."""
    pi = make_prerule_inputs(B=3, T=36, H=2, hk=1, dk=128, dv=128, dtype="f32", seed=57)
    ref = _oracle(pi)
    part = lambda s, e: type(pi)(**{**pi.__dict__, "x": pi.x[:, s:e], "a": pi.a[:, s:e], "b": pi.b[:, s:e]})
    (q, k, v, g, beta), hist = _run(part(0, 30))
    outs = [(q, k, v, g, beta)]
    for t in range(30, 36):
        st = part(t, t + 1)
        st.hist = hist.cpu()
        r, hist = _run(st, alias=True)
        outs.append(r)
    cat = [torch.cat([o[i] for o in outs], dim=1) for i in range(5)]
    _check(pi, cat, hist, ref)


def test_layer_core_end_to_end():
    """Raw projections -> gdn_prerule -> gdn_chunk_fwd equals the pre-rule oracle
    followed by the recurrence oracle (bf16, 16 value heads on 8 q/k heads)."""
    pi = make_prerule_inputs(B=2, T=300, H=16, hk=8, dk=128, dv=128, dtype="bf16", history=False, seed=58)
    (q, k, v, g, beta), _ = _run(pi, hist_out=False)
    out, fin, _ = gdn.gdn_chunk_fwd(q, k, v, g, beta)
    torch.cuda.synchronize()
    rq, rk, rv, rg, rb, _ = _oracle(pi)
    # the recurrence oracle takes the pre-rule results rounded as the library stores them
    bf = lambda z: torch.from_numpy(z).to(torch.bfloat16)
    rep = lambda z: z.repeat_interleave(2, dim=2)
    o_ref, f_ref, _ = oracle.gated_delta_rule(rep(bf(rq)), rep(bf(rk)), bf(rv), torch.from_numpy(rg).float(),
                                              torch.from_numpy(rb).float())
    assert rel_l2(out, o_ref) <= 2e-2 and rel_l2(fin, f_ref) <= 1e-2


# ---------------------------------------------------------------------------
# gdn_decode_step_prerule: the pre-rule work and the decode step in one kernel
# ---------------------------------------------------------------------------

def _fused_decode_case(dtype, d, K, hk, H, T=6, history=True, seed=60):
    pi = make_prerule_inputs(B=5, T=T, H=H, hk=hk, dk=d, dv=d, K=K, dtype=dtype, history=history, seed=seed)
    rng = np.random.default_rng(seed + 1000)
    h0 = rng.normal(0.0, 0.02, size=(5, H, d, d)).astype(np.float32)
    dev = lambda t: t.cuda().contiguous()
    conv = dev(pi.hist) if pi.hist is not None else None
    state = torch.from_numpy(h0).cuda()
    outs = []
    for t in range(T):
        outs.append(gdn.gdn_decode_step_prerule(dev(pi.x[:, t]), dev(pi.a[:, t]), dev(pi.b[:, t]), dev(pi.conv_w),
                                                dev(pi.A_log), dev(pi.dt_bias), conv, state, hk=hk, dk=d, H=H,
                                                dv=d))
    torch.cuda.synchronize()
    # oracle: the pre-rule work over the T tokens, then the recurrence (q/k heads repeated
    # for the value heads that share them)
    rq, rk, rv, rg, rb, rhist = _oracle(pi)
    rep = lambda z: np.repeat(z, H // hk, axis=2)
    o_ref, f_ref, _ = oracle.gated_delta_rule(rep(rq), rep(rk), rv, rg, rb, h0)
    return torch.stack(outs, 1), state, conv, o_ref, f_ref, rhist


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("K", [4, 2])
@pytest.mark.parametrize("hk", [2, 4])  # shared query/key heads (history moved by a second kernel) or not
def test_fused_decode_steps(dtype, d, K, hk):
    out, state, conv, o_ref, f_ref, rhist = _fused_decode_case(dtype, d, K, hk=hk, H=4, seed=60 + K)
    tol_o, tol_s = (1e-4, 1e-4) if dtype == "f32" else (2e-2, 1e-2)
    assert rel_l2(out, o_ref) <= tol_o
    assert rel_l2(state, f_ref) <= tol_s
    assert np.array_equal(conv.cpu().double().numpy(), rhist)  # the history: raw inputs, copied exactly


def test_fused_decode_without_history_and_k1():
    # without a history every step sees zeros before its token: one step equals a
    # one-token sequence with no history
    out, state, conv, o_ref, f_ref, _ = _fused_decode_case("bf16", 128, 4, hk=1, H=2, T=1, history=False, seed=66)
    assert conv is None
    assert rel_l2(out, o_ref) <= 2e-2 and rel_l2(state, f_ref) <= 1e-2
    out, state, conv, o_ref, f_ref, _ = _fused_decode_case("f32", 64, 1, hk=2, H=2, seed=67)  # no history kept
    assert rel_l2(out, o_ref) <= 1e-4 and rel_l2(state, f_ref) <= 1e-4


def test_fused_decode_equals_prerule_then_decode():
    """The fused step and gdn_prerule followed by gdn_decode_step agree (fp32 inputs:
    the unfused path stores q, k, v in fp32 too)."""
    pi = make_prerule_inputs(B=4, T=1, H=4, hk=2, dk=128, dv=128, K=4, dtype="f32", seed=68)
    rng = np.random.default_rng(69)
    h0 = torch.from_numpy(rng.normal(0.0, 0.02, size=(4, 4, 128, 128)).astype(np.float32)).cuda()
    dev = lambda t: t.cuda().contiguous()
    s1, s2 = h0.clone(), h0.clone()
    c1, c2 = dev(pi.hist), dev(pi.hist)
    o1 = gdn.gdn_decode_step_prerule(dev(pi.x[:, 0]), dev(pi.a[:, 0]), dev(pi.b[:, 0]), dev(pi.conv_w),
                                     dev(pi.A_log), dev(pi.dt_bias), c1, s1, hk=2, dk=128, H=4, dv=128)
    q, k, v, g, beta = gdn.gdn_prerule(dev(pi.x), dev(pi.a), dev(pi.b), dev(pi.conv_w), dev(pi.A_log),
                                       dev(pi.dt_bias), hk=2, dk=128, H=4, dv=128, conv_state_in=c2,
                                       conv_state_out=c2)
    rep = lambda z: z.repeat_interleave(2, dim=2)
    o2 = gdn.gdn_decode_step(rep(q), rep(k), v, g, beta, s2)
    torch.cuda.synchronize()
    assert rel_l2(o1, o2.reshape(o1.shape).cpu().double().numpy()) <= 1e-5
    assert rel_l2(s1, s2.cpu().double().numpy()) <= 1e-5
    assert torch.equal(c1, c2)
