"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, on the
same seeded inputs, element by element (relative L2 over whole tensors).

Tolerances: 1e-4 for fp32 inputs; 2e-2 on outputs and 1e-2 on states and
snapshots for bf16 inputs with an fp32 state."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import (DECODE, KDA_PACKED, LONG_SNAPSHOTS, PREFILL_BF16, TINY_F32,
                                             Workload, make_inputs)
from gated_delta_rule_64_b200.inputs import Inputs
from tests.gpu_util import check, rel_l2, run_gpu, run_oracle, to_dev, tolerances

pytestmark = pytest.mark.gpu

def fresh(t):
    """A freshly allocated contiguous copy (slices of packed tensors are views whose
    start need not be 16-byte aligned, which the library requires)."""
    return torch.empty_like(t, memory_format=torch.contiguous_format).copy_(t)


SMALL = Workload("small", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=11)


def test_tiny_f32_workload():
    check(make_inputs(TINY_F32))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64), (64, 128)])
def test_shapes(dtype, per_channel, dk, dv):
    check(make_inputs(SMALL.replace(dtype=dtype, per_channel=per_channel, dk=dk, dv=dv)))


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65, 128, 129])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("per_channel", [False, True])
def test_lengths_around_the_chunk(T, dtype, per_channel):
    check(make_inputs(SMALL.replace(T=T, dtype=dtype, per_channel=per_channel, seed=T)))


def test_zero_length_copies_initial_state():
    x = make_inputs(SMALL.replace(T=0, dtype="f32"))
    dx = to_dev(x)
    out, fin, _ = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0)
    torch.cuda.synchronize()
    assert torch.equal(fin.cpu(), x.h0)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("per_channel", [False, True])
def test_packed_sequences(dtype, per_channel):
    lengths = [1, 63, 64, 65, 130, 0, 7, 200]
    w = SMALL.replace(dtype=dtype, per_channel=per_channel, seed=5)
    check(make_inputs(w, lengths=lengths))


@pytest.mark.parametrize("per_channel", [False, True])
def test_packed_stage_ring(per_channel):
    # bf16 (tensor-core path): sequences of 4 to 9 chunks with ragged tails, so the
    # scan's three operand stages wrap several times and the copy issued ahead of
    # each chunk meets every stage, next to empty and one-token sequences
    lengths = [257, 0, 449, 1, 320, 575, 193]
    w = SMALL.replace(per_channel=per_channel, seed=21)
    check(make_inputs(w, lengths=lengths))


@pytest.mark.parametrize("per_channel", [False, True])
def test_zero_length_bf16_copies_initial_state(per_channel):
    x = make_inputs(SMALL.replace(T=0, per_channel=per_channel, seed=22))
    dx = to_dev(x)
    out, fin, _ = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0)
    torch.cuda.synchronize()
    assert out.numel() == 0
    assert torch.equal(fin.cpu(), x.h0)


@pytest.mark.parametrize("n_seqs", [1, 3, 8, 37, 1000, 2049])
def test_packed_sequence_order(n_seqs):
    # the chunk table that a packed call writes near the start of its workspace: the
    # first global chunk of every sequence, then the sequences by decreasing chunk
    # count (ties in index order) that the scan's blocks take in launch order;
    # batches of more than 2048 sequences keep their own order
    rng = np.random.default_rng(n_seqs)
    lengths = rng.integers(0, 300, size=n_seqs)
    lengths[rng.random(n_seqs) < 0.2] = 64 * rng.integers(0, 4)  # ties, empty sequences
    w = Workload("order", B=1, T=0, H=1, dk=128, dv=128, dtype="bf16", h0_std=0.0, seed=n_seqs)
    x = make_inputs(w, lengths=[int(v) for v in lengths])
    dx = to_dev(x)
    nbytes = gdn.gdn_chunk_workspace_size(1, int(lengths.sum()), 1, 128, 128, n_seqs)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, None, dx.cu_seqlens, workspace=ws)
    torch.cuda.synchronize()
    # (after the 256-byte slot of the status word)
    table = ws[256: 256 + 4 * (2 * n_seqs + 1)].cpu().view(torch.int32).numpy().astype(np.int64)
    off, order = table[: n_seqs + 1], table[n_seqs + 1:]
    chunks = (lengths + 63) // 64
    assert off[0] == 0 and np.array_equal(np.diff(off), chunks)
    if n_seqs > 2048:
        assert np.array_equal(order, np.arange(n_seqs))
    else:
        expect = sorted(range(n_seqs), key=lambda i: (-chunks[i], i))
        assert np.array_equal(order, expect)


def test_packed_equals_separate_runs():
    lengths = [70, 129, 3]
    x = make_inputs(SMALL.replace(seed=6), lengths=lengths)
    out, fin, _ = run_gpu(x)
    cu = x.cu_seqlens.tolist()
    for n in range(len(lengths)):
        a, b = cu[n], cu[n + 1]
        dx = to_dev(x)
        o1, f1, _ = gdn.gdn_chunk_fwd(fresh(dx.q[:, a:b]), fresh(dx.k[:, a:b]), fresh(dx.v[:, a:b]),
                                      fresh(dx.g[:, a:b]), fresh(dx.beta[:, a:b]),
                                      fresh(dx.h0[n:n + 1]))
        assert rel_l2(o1, out[:, a:b].cpu().double().numpy()) < 1e-6
        assert rel_l2(f1, fin[n:n + 1].cpu().double().numpy()) < 1e-6


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("per_channel", [False, True])
def test_snapshots(dtype, per_channel):
    x = make_inputs(SMALL.replace(T=640, dtype=dtype, per_channel=per_channel, seed=7))
    check(x, snapshot_stride=128)


def test_snapshot_resume_equals_full_run():
    x = make_inputs(SMALL.replace(T=512, dtype="f32", seed=8))
    dx = to_dev(x)
    out, fin, snaps = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0, snapshot_stride=192)
    n = 192
    o2, f2, _ = gdn.gdn_chunk_fwd(fresh(dx.q[:, n:]), fresh(dx.k[:, n:]), fresh(dx.v[:, n:]),
                                  fresh(dx.g[:, n:]), fresh(dx.beta[:, n:]), fresh(snaps[:, 0]))
    assert rel_l2(o2, out[:, n:].cpu().double().numpy()) < 1e-5
    assert rel_l2(f2, fin.cpu().double().numpy()) < 1e-5


def test_final_state_may_alias_initial_state():
    x = make_inputs(SMALL.replace(dtype="f32", seed=9))
    o_ref, f_ref, _ = run_oracle(x)
    dx = to_dev(x)
    st = dx.h0.clone()
    out, fin, _ = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, st, final_state=st)
    torch.cuda.synchronize()
    assert fin.data_ptr() == st.data_ptr()
    assert rel_l2(st, f_ref) <= 1e-4 and rel_l2(out, o_ref) <= 1e-4


def test_query_scale():
    check(make_inputs(SMALL.replace(seed=10)), scale=0.125)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("per_channel", [False, True])
def test_long_memory_gates(dtype, per_channel):
    """alpha ~ 0.999 and weak writes: the state and the initial state carry
    across many chunks."""
    w = SMALL.replace(T=2048, H=2, dtype=dtype, per_channel=per_channel, gate_mu=-7.0, beta_mu=-4.0, h0_std=0.3,
                      seed=12)
    check(make_inputs(w))


def _with_gates(x, g):
    x.g = g
    return x


def test_extreme_gates_scalar():
    """alpha = 1 (g = 0) with full-strength writes, and g = -80 on some tokens."""
    x = make_inputs(SMALL.replace(dtype="f32", seed=13))
    g = torch.zeros_like(x.g)
    g[:, 100:110] = -80.0
    x.beta = torch.ones_like(x.beta)
    check(_with_gates(x, g))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_extreme_gates_per_channel(dtype):
    """Per-channel gates mixing 0 and -80, with in-chunk gate sums far below the
    fp32 exponent range: nothing may overflow."""
    x = make_inputs(SMALL.replace(dtype=dtype, per_channel=True, seed=14))
    g = torch.zeros_like(x.g)
    g[..., ::3] = -80.0
    g[:, 50:60, :, 1::3] = -5.0
    check(_with_gates(x, g))


def test_per_channel_gate_strength_by_chunk():
    """Per-channel gates whose strength changes from chunk to chunk, so one launch
    forms A and P in every way the prep has: chunk 0 ordinary gates and chunk 3
    g = -1.2 per token (one product; 55 of the 60 log2 units it allows), chunk 1
    g = -1.5 (blocks: 69 units), chunk 2 g = -80 on every fourth channel (blocks
    with the diagonal blocks term by term), chunk 4 ordinary again."""
    x = make_inputs(SMALL.replace(T=320, H=2, per_channel=True, seed=23))
    g = x.g.clone()
    g[:, 64:128] = -1.5
    g[:, 128:192, :, ::4] = -80.0
    g[:, 192:256] = -1.2
    check(_with_gates(x, g))


@pytest.mark.parametrize("gate_mu", [2.0, 6.0])
def test_strong_per_channel_gates(gate_mu):
    """Strong decays on every channel (alpha ~ e^-2 .. e^-6 per token): in-chunk
    cumulative gates of several hundred, far outside the fp32 range of exp."""
    check(make_inputs(SMALL.replace(per_channel=True, gate_mu=gate_mu, seed=15)))


@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("gate_mu", [-2.0, -7.0])
def test_split_scan(per_channel, gate_mu):
    """One long sequence on two heads (128 chunks): the scan splits it into segments
    (state maps per segment, chained start states); gate_mu = -7 keeps the state
    alive across every segment boundary."""
    w = SMALL.replace(B=1, T=8192, H=2, per_channel=per_channel, gate_mu=gate_mu, h0_std=0.1, seed=16)
    check(make_inputs(w), snapshot_stride=1024)


def test_split_scan_final_state_aliases_initial():
    w = SMALL.replace(B=1, T=8192, H=2, h0_std=0.1, seed=17)
    x = make_inputs(w)
    dx = to_dev(x)
    st = dx.h0.clone()
    out, fin, _ = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, st, final_state=st)
    torch.cuda.synchronize()
    o_ref, f_ref, _ = run_oracle(x)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert fin.data_ptr() == st.data_ptr()
    assert rel_l2(out, o_ref) <= tol_o and rel_l2(st, f_ref) <= tol_s


# ---------------------------------------------------------------------------
# Decode
# ---------------------------------------------------------------------------

def _decode_oracle(x):
    """Steps as a sequence per (b, h): (steps, B, 1, H, .) -> (B, steps, H, .)."""
    seq = lambda t: t[:, :, 0].transpose(0, 1)
    return oracle.gated_delta_rule(seq(x.q), seq(x.k), seq(x.v), seq(x.g), seq(x.beta), x.h0)


def _decode_gpu(x):
    dx = to_dev(x)
    state = dx.h0.clone()
    outs = [gdn.gdn_decode_step(dx.q[s], dx.k[s], dx.v[s], dx.g[s], dx.beta[s], state) for s in range(x.q.shape[0])]
    # (per-step slices of the gates start on 4-byte boundaries only, which the library accepts)
    torch.cuda.synchronize()
    return torch.stack([o[:, 0] for o in outs], 1), state


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_decode_steps(dtype, per_channel, dk, dv):
    w = DECODE.replace(B=6, H=3, dk=dk, dv=dv, decode_steps=20, dtype=dtype, per_channel=per_channel, seed=20)
    x = make_inputs(w)
    o, s = _decode_gpu(x)
    o_ref, s_ref, _ = _decode_oracle(x)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(o, o_ref) <= tol_o and rel_l2(s, s_ref) <= tol_s


def test_decode_continues_prefill():
    """Prefill of T tokens then decode of more equals prefill of all of them."""
    w = SMALL.replace(T=200, dtype="f32", seed=21)
    x = make_inputs(w)
    dx = to_dev(x)
    P = 150
    _, st, _ = gdn.gdn_chunk_fwd(fresh(dx.q[:, :P]), fresh(dx.k[:, :P]), fresh(dx.v[:, :P]),
                                 fresh(dx.g[:, :P]), fresh(dx.beta[:, :P]), dx.h0)
    outs = []
    for t in range(P, 200):
        outs.append(gdn.gdn_decode_step(fresh(dx.q[:, t:t + 1]), fresh(dx.k[:, t:t + 1]),
                                        fresh(dx.v[:, t:t + 1]), fresh(dx.g[:, t:t + 1]),
                                        fresh(dx.beta[:, t:t + 1]), st)[:, 0])
    out_all, fin_all, _ = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0)
    torch.cuda.synchronize()
    assert rel_l2(torch.stack(outs, 1), out_all[:, P:].cpu().double().numpy()) < 1e-4
    assert rel_l2(st, fin_all.cpu().double().numpy()) < 1e-4


# ---------------------------------------------------------------------------
# Multi-token decode (speculative verify) and rollback
# ---------------------------------------------------------------------------

def _multi_inputs(dtype, per_channel, d, B=5, T=6, H=3, seed=30, dv=None):
    w = DECODE.replace(B=B, H=H, dk=d, dv=d if dv is None else dv, decode_steps=0, T=T, dtype=dtype,
                       per_channel=per_channel, h0_std=0.1, seed=seed)
    return make_inputs(w)


def _multi_oracle(x, n):
    """Per sequence b: its first n[b] tokens from its own initial state, with the
    state after every token (snapshot stride 1)."""
    B = x.q.shape[0]
    outs, finals, steps = [], [], []
    for b in range(B):
        nb = int(n[b])
        sl = lambda t: t[b:b + 1, :nb]
        if nb == 0:
            outs.append(None); finals.append(x.h0[b].double().numpy()); steps.append(None)
            continue
        o, f, sn = oracle.gated_delta_rule(sl(x.q), sl(x.k), sl(x.v), sl(x.g), sl(x.beta), x.h0[b:b + 1],
                                           snapshot_stride=1)
        outs.append(o[0]); finals.append(f[0]); steps.append(sn[0])
    return outs, finals, steps


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("per_channel", [False, True])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (128, 64), (64, 128)])
def test_decode_multi_commit(dtype, per_channel, dk, dv):
    x = _multi_inputs(dtype, per_channel, dk, dv=dv)
    dx = to_dev(x)
    st = dx.h0.clone()
    out, steps = gdn.gdn_decode_multi(dx.q, dx.k, dx.v, dx.g, dx.beta, st, commit=True, step_states=True)
    torch.cuda.synchronize()
    B, T = x.q.shape[:2]
    o_ref, f_ref, s_ref = _multi_oracle(x, [T] * B)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(out, np.stack(o_ref)) <= tol_o
    assert rel_l2(st, np.stack(f_ref)) <= tol_s
    assert rel_l2(steps, np.stack(s_ref)) <= tol_s


@pytest.mark.parametrize("per_channel", [False, True])
def test_decode_multi_rollback(per_channel):
    """Verify drafts without committing (the pre-draft state stays bit for bit),
    then adopt the state after each sequence's accepted prefix."""
    x = _multi_inputs("bf16", per_channel, 128, B=6, T=8, seed=31)
    dx = to_dev(x)
    n = torch.tensor([0, 3, 8, 1, 5, 8], dtype=torch.int32)
    st = dx.h0.clone()
    out, steps = gdn.gdn_decode_multi(dx.q, dx.k, dx.v, dx.g, dx.beta, st, n_tokens=n.cuda(), commit=False,
                                      step_states=True)
    torch.cuda.synchronize()
    assert torch.equal(st, dx.h0)
    o_ref, f_ref, s_ref = _multi_oracle(x, n.tolist())
    tol_o, tol_s = tolerances(x.q.dtype)
    for b, nb in enumerate(n.tolist()):
        if nb:
            assert rel_l2(out[b, :nb], o_ref[b]) <= tol_o
            assert rel_l2(steps[b, :nb], s_ref[b]) <= tol_s
    accept = torch.tensor([0, 2, 8, 1, 0, 4], dtype=torch.int32)
    gdn.gdn_state_select(steps, accept.cuda(), st)
    # the same states by committing only the accepted tokens from the pre-draft state
    st2 = dx.h0.clone()
    gdn.gdn_decode_multi(dx.q, dx.k, dx.v, dx.g, dx.beta, st2, n_tokens=accept.cuda(), commit=True)
    torch.cuda.synchronize()
    assert torch.equal(st, st2)
    _, f_acc, _ = _multi_oracle(x, accept.tolist())
    assert rel_l2(st, np.stack(f_acc)) <= tol_s


def test_decode_multi_equals_single_steps():
    x = _multi_inputs("f32", False, 128, B=4, T=5, seed=32)
    dx = to_dev(x)
    st = dx.h0.clone()
    out, _ = gdn.gdn_decode_multi(dx.q, dx.k, dx.v, dx.g, dx.beta, st)
    st1 = dx.h0.clone()
    outs = [gdn.gdn_decode_step(fresh(dx.q[:, t:t + 1]), fresh(dx.k[:, t:t + 1]), fresh(dx.v[:, t:t + 1]),
                                fresh(dx.g[:, t:t + 1]), fresh(dx.beta[:, t:t + 1]), st1)[:, 0] for t in range(5)]
    torch.cuda.synchronize()
    assert rel_l2(out, torch.stack(outs, 1).cpu().double().numpy()) < 1e-6
    assert rel_l2(st, st1.cpu().double().numpy()) < 1e-6


# ---------------------------------------------------------------------------
# Shared query/key heads (fewer q/k heads than value heads)
# ---------------------------------------------------------------------------

def _share_qk(x, hk):
    """Keep the first hk query/key heads; the oracle sees them repeated so that
    value head h reads query/key head h // (H // hk)."""
    H = x.q.shape[-2]
    rep = lambda t: t.repeat_interleave(H // hk, dim=-2)
    q_small, k_small = x.q[..., :hk, :].contiguous(), x.k[..., :hk, :].contiguous()
    ref = Inputs(q=rep(q_small), k=rep(k_small), v=x.v, g=x.g, beta=x.beta, h0=x.h0, cu_seqlens=x.cu_seqlens,
                 workload=x.workload)
    gpu = Inputs(q=q_small, k=k_small, v=x.v, g=x.g, beta=x.beta, h0=x.h0, cu_seqlens=x.cu_seqlens,
                 workload=x.workload)
    return gpu, ref


@pytest.mark.parametrize("dtype,per_channel", [("bf16", False), ("bf16", True), ("f32", False), ("f32", True)])
@pytest.mark.parametrize("hk", [1, 2])
def test_shared_qk_heads_prefill(dtype, per_channel, hk):
    x = make_inputs(SMALL.replace(H=4, T=200, dtype=dtype, per_channel=per_channel, seed=40), lengths=None)
    gx, rx = _share_qk(x, hk)
    out, fin, _ = run_gpu(gx)
    o_ref, f_ref, _ = run_oracle(rx)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(out, o_ref) <= tol_o and rel_l2(fin, f_ref) <= tol_s


def test_shared_qk_heads_packed_and_split():
    # packed sequences, then one long fixed-length sequence (split scan), 4 value heads on 2 q/k heads
    x = make_inputs(SMALL.replace(H=4, seed=41), lengths=[70, 1, 300, 64])
    gx, rx = _share_qk(x, 2)
    out, fin, _ = run_gpu(gx)
    o_ref, f_ref, _ = run_oracle(rx)
    assert rel_l2(out, o_ref) <= 2e-2 and rel_l2(fin, f_ref) <= 1e-2
    x = make_inputs(SMALL.replace(B=1, T=8192, H=2, h0_std=0.1, seed=42))
    gx, rx = _share_qk(x, 1)
    out, fin, snaps = run_gpu(gx, snapshot_stride=2048)
    o_ref, f_ref, s_ref = run_oracle(rx, snapshot_stride=2048)
    assert rel_l2(out, o_ref) <= 2e-2 and rel_l2(fin, f_ref) <= 1e-2 and rel_l2(snaps, s_ref) <= 1e-2


@pytest.mark.parametrize("per_channel", [False, True])
def test_shared_qk_heads_decode(per_channel):
    x = _multi_inputs("bf16", per_channel, 128, B=4, T=5, H=4, seed=43)
    gx, rx = _share_qk(x, 2)
    dx = to_dev(gx)
    st = dx.h0.clone()
    out, steps = gdn.gdn_decode_multi(dx.q, dx.k, dx.v, dx.g, dx.beta, st, step_states=True)
    st1 = dx.h0.clone()
    out1 = gdn.gdn_decode_step(fresh(dx.q[:, :1]), fresh(dx.k[:, :1]), fresh(dx.v[:, :1]), fresh(dx.g[:, :1]),
                               fresh(dx.beta[:, :1]), st1)
    torch.cuda.synchronize()
    o_ref, f_ref, s_ref = _multi_oracle(rx, [5] * 4)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(out, np.stack(o_ref)) <= tol_o and rel_l2(st, np.stack(f_ref)) <= tol_s
    assert rel_l2(out1[:, 0], np.stack(o_ref)[:, 0]) <= tol_o
    assert rel_l2(st1, np.stack(s_ref)[:, 0]) <= tol_s


# ---------------------------------------------------------------------------
# The benchmark workloads at full size (oracle on sampled heads / sequences)
# ---------------------------------------------------------------------------

def _per_unit_report(name, errs):
    """Largest per-(sequence, head) relative L2 error of each tensor, appended to the
    optional parity report."""
    import os
    report = os.environ.get("GDN_PARITY_REPORT")
    if report:
        with open(report, "a") as f:
            f.write(f"{name}\tper-(sequence, head) max\t" + "\t".join(f"{k} {v:.3e}" for k, v in errs.items()) + "\n")


def _check_every_unit(x, snapshot_stride=0):
    """Every (sequence, head) of a full-size workload: whole tensors and each
    (sequence, head) slice against the oracle."""
    out, fin, snaps = run_gpu(x, snapshot_stride=snapshot_stride)
    o_ref, f_ref, s_ref = run_oracle(x, snapshot_stride=snapshot_stride)
    tol_o, tol_s = tolerances(x.q.dtype)
    assert rel_l2(out, o_ref) <= tol_o and rel_l2(fin, f_ref) <= tol_s
    if snapshot_stride:
        assert rel_l2(snaps, s_ref) <= tol_s
    out, fin = out.cpu(), fin.cpu()
    H = x.v.shape[2]
    cu = x.cu_seqlens.tolist() if x.cu_seqlens is not None else None
    worst = {"out": 0.0, "state": 0.0, "snapshots": 0.0}
    for n in range(fin.shape[0]):
        for h in range(H):
            if cu is None:
                eo = rel_l2(out[n, :, h], o_ref[n, :, h])
            else:
                eo = rel_l2(out[0, cu[n]:cu[n + 1], h], o_ref[0, cu[n]:cu[n + 1], h]) if cu[n + 1] > cu[n] else 0.0
            ef = rel_l2(fin[n, h], f_ref[n, h])
            es = rel_l2(snaps[n, :, h].cpu(), s_ref[n, :, h]) if snapshot_stride else 0.0
            assert eo <= tol_o and ef <= tol_s and es <= tol_s, (n, h, eo, ef, es)
            worst = {"out": max(worst["out"], eo), "state": max(worst["state"], ef),
                     "snapshots": max(worst["snapshots"], es)}
    return worst


def test_prefill_workload_full_size():
    _per_unit_report("prefill B4 T4096 H16 (all 64 sequence-heads)", _check_every_unit(make_inputs(PREFILL_BF16)))


def test_long_snapshot_workload_full_size():
    x = make_inputs(LONG_SNAPSHOTS)
    _per_unit_report("long T262144 H16 snapshots/8192 (all 16 heads)",
                     _check_every_unit(x, snapshot_stride=LONG_SNAPSHOTS.snapshot_stride))


def test_kda_packed_workload_full_size():
    _per_unit_report("kda packed 8 sequences H32 (all 256 sequence-heads)", _check_every_unit(make_inputs(KDA_PACKED)))


def test_decode_workload_full_size():
    """All 256 sequences x 32 heads over the 64 steps, each (sequence, head) too."""
    x = make_inputs(DECODE)
    o, s = _decode_gpu(x)
    o_ref, s_ref, _ = _decode_oracle(x)
    assert rel_l2(o, o_ref) <= 2e-2 and rel_l2(s, s_ref) <= 1e-2
    o, s = o.cpu(), s.cpu()
    worst_o = max(rel_l2(o[b, :, h], o_ref[b, :, h]) for b in range(o.shape[0]) for h in range(o.shape[2]))
    worst_s = max(rel_l2(s[b, h], s_ref[b, h]) for b in range(s.shape[0]) for h in range(s.shape[1]))
    assert worst_o <= 2e-2 and worst_s <= 1e-2
    _per_unit_report("decode 256 x H32, 64 steps (all 8192 sequence-heads)", {"out": worst_o, "state": worst_s})
