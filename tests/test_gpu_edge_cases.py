"""GPU parity on the cases the pages single out, on the benchmarked path.

The chunked prefill with bf16 q/k/v and d = 128 runs on the tensor cores
(gdn_prep_tc / gdn_scan_tc, and the per-channel kernels); decode runs the
streaming step kernels.  Each case below is compared element by element with the
fp64 oracle at the usual tolerances (bf16: 2e-2 on outputs, 1e-2 on states),
and where the pages give a closed form, with that too:

  beta = 0        only the decay acts ("pure forgetting": "From Traditional
                  Attention to hybrid ones", section 5): the final state is
                  (prod alpha) S0, per key channel for the per-channel gate;
  beta = 1, g = 0 the DeltaNet rule (alpha = 1, full-strength writes: same page,
                  section 5; "Attention, Part 4", section 4);
  g = -80         a run of tokens whose decay wipes the state (alpha = e^-80),
                  across a chunk boundary;
  g = 0           whole chunks without decay between ordinary ones.

Every case starts from a non-zero initial state and spans several chunks; the
split scan (one long sequence) is run on the same cases.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import DECODE, Workload, make_inputs
from tests.gpu_util import rel_l2, run_gpu, run_oracle, tolerances, to_dev

pytestmark = pytest.mark.gpu

BASE = Workload("edge", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=70)
LONG = Workload("edge long", B=1, T=8192, H=2, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=71)
CASES = ["beta0", "delta", "g-80", "g0-chunks"]


def _edit(x, case):
    """Apply a case to freshly drawn inputs (token axis 1 of (B, T, H[, dk]))."""
    T = x.g.shape[1]
    if case == "beta0":
        x.beta = torch.zeros_like(x.beta)
    elif case == "delta":
        x.beta = torch.ones_like(x.beta)
        x.g = torch.zeros_like(x.g)
    elif case == "g-80":
        g = x.g.clone()
        g[:, 60:70] = -80.0  # across the boundary of the first two chunks
        if T > 4096:
            g[:, 4090:4100] = -80.0
        x.g = g
    elif case == "g0-chunks":
        g = x.g.clone()
        for c0 in range(64, T, 128):  # every other chunk without decay
            g[:, c0:c0 + 64] = 0.0
        x.g = g
    return x


def _closed_form_beta0(x, fin):
    """beta = 0: S_T = S0 Diag(exp(sum_t g_t)) (a scalar per head for one gate per head)."""
    G = x.g.double().sum(1)  # (B, H) or (B, H, dk)
    h0 = x.h0.double()
    ref = h0 * torch.exp(G)[..., None, None] if G.dim() == 2 else h0 * torch.exp(G)[:, :, None, :]
    assert rel_l2(fin, ref.numpy()) <= 1e-2


@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_prefill_tensor_cores(case, per_channel):
    x = _edit(make_inputs(BASE.replace(per_channel=per_channel)), case)
    out, fin, snaps = run_gpu(x, snapshot_stride=128)
    o_ref, f_ref, s_ref = run_oracle(x, snapshot_stride=128)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(out, o_ref) <= tol_o
    assert rel_l2(fin, f_ref) <= tol_s and rel_l2(snaps, s_ref) <= tol_s
    if case == "beta0":
        _closed_form_beta0(x, fin)


@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_prefill_split_scan(case, per_channel):
    """One sequence of 128 chunks: the scan splits it; "delta" and "g0-chunks" keep
    the start state alive through every segment (transition maps, whole segments
    rerun), "beta0" with ordinary gates and "g-80" forget it (short rerun)."""
    x = _edit(make_inputs(LONG.replace(per_channel=per_channel)), case)
    out, fin, snaps = run_gpu(x, snapshot_stride=1024)
    o_ref, f_ref, s_ref = run_oracle(x, snapshot_stride=1024)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(out, o_ref) <= tol_o
    assert rel_l2(fin, f_ref) <= tol_s and rel_l2(snaps, s_ref) <= tol_s
    if case == "beta0":
        _closed_form_beta0(x, fin)


def _decode_case(case, per_channel, steps=20):
    w = DECODE.replace(B=6, H=3, decode_steps=steps, per_channel=per_channel, h0_std=0.1, seed=72)
    x = make_inputs(w)
    # steps play the role of tokens: (steps, B, 1, H[, dk]) -> edit along the step axis
    if case == "beta0":
        x.beta = torch.zeros_like(x.beta)
    elif case == "delta":
        x.beta = torch.ones_like(x.beta)
        x.g = torch.zeros_like(x.g)
    elif case == "g-80":
        x.g = x.g.clone()
        x.g[5:9] = -80.0
    elif case == "g0-chunks":
        x.g = x.g.clone()
        x.g[4:12] = 0.0
    return x


def _decode_oracle(x):
    seq = lambda t: t[:, :, 0].transpose(0, 1)
    return run_oracle_seq(seq(x.q), seq(x.k), seq(x.v), seq(x.g), seq(x.beta), x.h0)


def run_oracle_seq(q, k, v, g, beta, h0):
    import oracle
    return oracle.gated_delta_rule(q, k, v, g, beta, h0)


@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_decode_step(case, per_channel):
    x = _decode_case(case, per_channel)
    dx = to_dev(x)
    state = dx.h0.clone()
    outs = [gdn.gdn_decode_step(dx.q[s], dx.k[s], dx.v[s], dx.g[s], dx.beta[s], state) for s in range(x.q.shape[0])]
    torch.cuda.synchronize()
    o = torch.stack([t[:, 0] for t in outs], 1)
    o_ref, s_ref, _ = _decode_oracle(x)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(o, o_ref) <= tol_o and rel_l2(state, s_ref) <= tol_s


@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("case", CASES)
def test_decode_multi(case, per_channel):
    """The same cases as one multi-token call per sequence (12 tokens), committed,
    with every step's state."""
    x = _decode_case(case, per_channel, steps=12)
    seq = lambda t: t[:, :, 0].transpose(0, 1).contiguous()  # (B, T, H[, dk])
    q, k, v, g, beta = (seq(t) for t in (x.q, x.k, x.v, x.g, x.beta))
    d = lambda t: t.cuda()
    st = d(x.h0).clone()
    out, steps = gdn.gdn_decode_multi(d(q), d(k), d(v), d(g), d(beta), st, commit=True, step_states=True)
    torch.cuda.synchronize()
    import oracle
    o_ref, f_ref, s_ref = oracle.gated_delta_rule(q, k, v, g, beta, x.h0, snapshot_stride=1)
    tol_o, tol_s = tolerances(q.dtype)
    assert rel_l2(out, o_ref) <= tol_o
    assert rel_l2(st, f_ref) <= tol_s and rel_l2(steps, s_ref) <= tol_s


def test_carry_stress_split_scan():
    """Gates that keep the state alive for thousands of tokens (alpha ~ 0.999, weak
    writes, large initial state) on one sequence of 65,536 tokens: the scan splits it
    into many segments whose transition maps are all needed and chained, and every
    snapshot (each 8,192 tokens) and output is checked."""
    w = Workload("carry stress", B=1, T=65536, H=1, dk=128, dv=128, dtype="bf16", gate_mu=-7.0, beta_mu=-4.0,
                 h0_std=0.3, seed=73)
    x = make_inputs(w)
    out, fin, snaps = run_gpu(x, snapshot_stride=8192)
    o_ref, f_ref, s_ref = run_oracle(x, snapshot_stride=8192)
    tol_o, tol_s = tolerances(x.q.dtype)
    eo, ef, es = rel_l2(out, o_ref), rel_l2(fin, f_ref), rel_l2(snaps, s_ref)
    assert eo <= tol_o and ef <= tol_s and es <= tol_s, (eo, ef, es)
    # for this test to mean anything the start state of every 2,048-token stretch
    # must still matter at its end (far above the 2^-126 bound where it is dropped)
    lam = x.g.double()[0, :, 0].numpy().reshape(-1, 2048).sum(1) / np.log(2.0)
    assert lam.min() > -60.0
