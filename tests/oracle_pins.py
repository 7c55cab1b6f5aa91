"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Each ``pin_*`` function takes ``run`` (the oracle entry point, or a build of
it with a planted mistake) and raises AssertionError when the oracle disagrees
with a value printed on the pages, a closed form, an identity or a brute-force
evaluation.  None of them re-types the oracle's loop: each computes the
expected value by a different route (a printed number, a product of matrices,
a masked parallel form, autograd, a cumulative-log closed form ...).
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit(a):
    return a / np.linalg.norm(a, axis=-1, keepdims=True)


def _rand_problem(seed, T, H=2, dk=5, dv=3, per_channel=False, B=1, gate_lo=-1.0, h0=True):
    r = _rng(seed)
    q = _unit(r.standard_normal((B, T, H, dk)))
    k = _unit(r.standard_normal((B, T, H, dk)))
    v = r.standard_normal((B, T, H, dv))
    beta = r.uniform(0.05, 0.95, (B, T, H))
    g = r.uniform(gate_lo, 0.0, (B, T, H, dk) if per_channel else (B, T, H))
    S0 = r.standard_normal((B, H, dv, dk)) * 0.5 if h0 else None
    return q, k, v, g, beta, S0


def _close(a, b, tol, what):
    a, b = np.asarray(a, dtype=np.float64), np.asarray(b, dtype=np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, float(np.max(np.abs(b)))) if b.size else 1.0
    assert err <= tol * scale, f"{what}: max|diff| {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------------------
# Printed values
# ---------------------------------------------------------------------------

def pin_decay_table(run):
    """beta = 0 leaves only the forget gate: a stored value fades as alpha**t.

    Printed table: "Attention, Part 4", section 5 (output 4)."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "decay_table.txt")) if l.strip() and l[0] != "#"]
    for alpha in sorted({float(r[0]) for r in rows}):
        T = 500
        one = np.ones((1, T, 1, 1))
        g = np.full((1, T, 1), math.log(alpha))
        out, _, _ = run(one, one, one, g, np.zeros((1, T, 1)), initial_state=np.ones((1, 1, 1, 1)))
        strength = {0: 1.0}
        strength.update({t: out[0, t - 1, 0, 0] for t in range(1, T + 1)})
        for a, t, val in rows:
            if float(a) == alpha:
                assert f"{strength[int(t)]:.3f}" == val, (alpha, t, strength[int(t)], val)


def pin_overwrite_example(run):
    """x = 1, y = 7, x = 5 with perpendicular keys: delta rule reads back (5, 7),
    plain adding (6, 7).  Printed: "Attention, Part 4", section 3, Test 1."""
    rows = {l.split()[0]: (l.split()[1], l.split()[2]) for l in open(os.path.join(GOLDEN, "overwrite_example.txt"))
            if l.strip() and l[0] != "#"}
    ex, ey = np.array([1.0, 0.0]), np.array([0.0, 1.0])
    keys = [ex, ey, ex, ex, ey]            # three writes, then two reads
    vals = [1.0, 7.0, 5.0, 0.0, 0.0]
    betas = [1.0, 1.0, 1.0, 0.0, 0.0]      # the reads write nothing
    T = len(keys)
    k = np.array(keys).reshape(1, T, 1, 2)
    q = k.copy()
    v = np.array(vals).reshape(1, T, 1, 1)
    beta = np.array(betas).reshape(1, T, 1)
    g = np.zeros((1, T, 1))                # alpha = 1: no forgetting
    for rule, additive in (("delta", False), ("linear", True)):
        out, _, _ = run(q, k, v, g, beta, additive=additive)
        got = (f"{out[0, 3, 0, 0]:.2f}", f"{out[0, 4, 0, 0]:.2f}")
        assert got == rows[rule], (rule, got, rows[rule])


# ---------------------------------------------------------------------------
# Closed forms and identities
# ---------------------------------------------------------------------------

def pin_beta_zero_is_pure_decay(run):
    """beta = 0: S_T = (prod alpha_t) S_0, or S_0 Diag(prod alpha_t) per channel
    ("From Traditional Attention to hybrid ones", sections 5 and 7)."""
    for per_channel in (False, True):
        q, k, v, g, beta, S0 = _rand_problem(1, T=9, per_channel=per_channel)
        _, fin, _ = run(q, k, v, g, np.zeros_like(beta), initial_state=S0)
        tot = np.exp(g.sum(axis=1))[0]     # (H,) or (H, dk)
        if per_channel:
            want = S0[0] * tot[:, None, :]  # scales the key channels (columns)
        else:
            want = S0[0] * tot[:, None, None]
        _close(fin[0], want, 1e-13, f"beta=0 decay per_channel={per_channel}")


def pin_read_after_write(run):
    """alpha = beta = 1 with unit keys: reading with the key just written
    returns its value exactly ("Attention, Part 4", section 4)."""
    q, k, v, g, beta, S0 = _rand_problem(2, T=12, dk=6, dv=4)
    out, _, _ = run(k, k, v, np.zeros_like(g), np.ones_like(beta), initial_state=S0)
    _close(out, v, 1e-13, "S_t k_t = v_t")


def pin_fixed_point(run):
    """A state that already maps k to v is left unchanged by the delta rule for
    any beta ("Hybrid models ...", section "The delta rule")."""
    r = _rng(3)
    dk, dv, H = 6, 4, 2
    k = _unit(r.standard_normal((1, 1, H, dk)))
    v = r.standard_normal((1, 1, H, dv))
    S0 = r.standard_normal((1, H, dv, dk))
    for h in range(H):
        S0[0, h] += np.outer(v[0, 0, h] - S0[0, h] @ k[0, 0, h], k[0, 0, h])  # now S0 k = v
    for b in (0.3, 0.9, 1.0):
        _, fin, _ = run(k, k, v, np.zeros((1, 1, H)), np.full((1, 1, H), b), initial_state=S0)
        _close(fin, S0, 1e-13, f"fixed point beta={b}")


def pin_linear_attention_parallel_form(run):
    """Additive writes, no gate: the output equals the masked parallel form
    tril(Q K^T) V ("Attention, Part 4", section 2; "Hybrid attention",
    "Attention without the softmax")."""
    q, k, v, g, beta, _ = _rand_problem(4, T=40, dk=7, dv=5, h0=False)
    out, fin, _ = run(q, k, v, np.zeros_like(g), np.ones_like(beta), additive=True)
    for h in range(q.shape[2]):
        Q, K, V = q[0, :, h], k[0, :, h], v[0, :, h]
        _close(out[0, :, h], np.tril(Q @ K.T) @ V, 1e-12, "linear attention parallel form")
        _close(fin[0, h], V.T @ K, 1e-12, "linear attention state = sum v k^T")


def pin_gated_additive_closed_form(run):
    """Additive writes with a forget gate (the Mamba-2 form S_t = alpha_t S_{t-1}
    + beta_t v_t k_t^T): o_t = prod_{j<=t} alpha_j S_0 q_t
    + sum_{i<=t} prod_{i<j<=t} alpha_j beta_i (q_t . k_i) v_i
    ("Attention, Part 4", section 5)."""
    q, k, v, g, beta, S0 = _rand_problem(5, T=30, dk=4, dv=3)
    out, _, _ = run(q, k, v, g, beta, initial_state=S0, additive=True)
    for h in range(q.shape[2]):
        c = np.cumsum(g[0, :, h])                          # log prod_{j<=t} alpha_j
        decay = np.exp(c[:, None] - c[None, :])            # prod_{i<j<=t} alpha_j
        M = np.tril((q[0, :, h] @ k[0, :, h].T) * decay) * beta[0, :, h][None, :]
        want = M @ v[0, :, h] + np.exp(c)[:, None] * (q[0, :, h] @ S0[0, h].T)
        _close(out[0, :, h], want, 1e-12, "gated additive closed form")


def _unrolled(q, k, v, g, beta, S0, per_channel):
    """S_t = S_0 M_1..M_t + sum_i beta_i v_i k_i^T M_{i+1}..M_t with
    M_t = alpha_t (I - beta_t k_t k_t^T), or Diag(alpha_t)(I - beta_t k_t k_t^T)
    per channel ("From Traditional Attention to hybrid ones", sections 5 and 7),
    evaluated as explicit matrix products."""
    T, dk = k.shape[0], k.shape[1]
    I = np.eye(dk)
    Ms = []
    for t in range(T):
        D = np.diag(np.exp(g[t])) if per_channel else np.exp(g[t]) * I
        Ms.append(D @ (I - beta[t] * np.outer(k[t], k[t])))
    outs, states = [], []
    for t in range(T):
        P = I.copy()
        for j in range(t + 1):
            P = P @ Ms[j]
        S = S0 @ P
        for i in range(t + 1):
            R = I.copy()
            for j in range(i + 1, t + 1):
                R = R @ Ms[j]
            S = S + beta[i] * np.outer(v[i], k[i]) @ R
        states.append(S)
        outs.append(S @ q[t])
    return np.array(outs), states[-1]


def pin_unrolled_product(run):
    """Brute force for T <= 8: the recurrence equals the unrolled product of
    its transition matrices, for the scalar and the per-channel gate."""
    for per_channel in (False, True):
        for T in (1, 3, 8):
            q, k, v, g, beta, S0 = _rand_problem(10 + T, T=T, per_channel=per_channel)
            out, fin, _ = run(q, k, v, g, beta, initial_state=S0)
            for h in range(q.shape[2]):
                o_ref, s_ref = _unrolled(q[0, :, h], k[0, :, h], v[0, :, h], g[0, :, h], beta[0, :, h],
                                         S0[0, h], per_channel)
                _close(out[0, :, h], o_ref, 1e-12, f"unrolled outputs T={T} pc={per_channel}")
                _close(fin[0, h], s_ref, 1e-12, f"unrolled state T={T} pc={per_channel}")


def pin_sgd_identity(run):
    """One step is one gradient step on 1/2 ||S k - v||^2 taken at the decayed
    state, step size beta ("Attention, Part 4", section 4; "Hybrid attention",
    "Writing with the delta rule").  The gradient comes from autograd."""
    q, k, v, g, beta, S0 = _rand_problem(20, T=1, dk=6, dv=4)
    _, fin, _ = run(q, k, v, g, beta, initial_state=S0)
    for h in range(q.shape[2]):
        St = torch.tensor(math.exp(g[0, 0, h]) * S0[0, h], dtype=torch.float64, requires_grad=True)
        kt = torch.tensor(k[0, 0, h]); vt = torch.tensor(v[0, 0, h])
        loss = 0.5 * torch.sum((St @ kt - vt) ** 2)
        loss.backward()
        want = (St - beta[0, 0, h] * St.grad).detach().numpy()
        _close(fin[0, h], want, 1e-13, "SGD identity")


def pin_orthonormal_capacity(run):
    """With d orthonormal keys, full write strength and no forgetting, the state
    after d writes is exactly sum v_i k_i^T ("Hybrid attention", "A memory of
    fixed size": orthogonal keys do not interfere)."""
    r = _rng(21)
    d, dv = 6, 4
    Qm, _ = np.linalg.qr(r.standard_normal((d, d)))
    k = Qm.T.reshape(1, d, 1, d)           # rows are orthonormal keys
    v = r.standard_normal((1, d, 1, dv))
    _, fin, _ = run(k, k, v, np.zeros((1, d, 1)), np.ones((1, d, 1)))
    _close(fin[0, 0], v[0, :, 0].T @ k[0, :, 0], 1e-13, "orthonormal capacity")


def pin_channel_gate_reduces_to_head_gate(run):
    """A per-channel gate with all channels equal is the scalar gate
    ("Attention, Part 4", section 7)."""
    q, k, v, g, beta, S0 = _rand_problem(22, T=17)
    gc = np.repeat(g[..., None], k.shape[-1], axis=-1)
    o1, f1, _ = run(q, k, v, g, beta, initial_state=S0)
    o2, f2, _ = run(q, k, v, gc, beta, initial_state=S0)
    _close(o1, o2, 1e-14, "KDA equal channels outputs")
    _close(f1, f2, 1e-14, "KDA equal channels state")


def pin_channel_gate_direction(run):
    """Per-channel forgetting scales key channels (columns of the d_v x d_k
    state), not value channels: with one key channel gated to ~0 before a write
    on an orthogonal key, that column of S_0 is gone and the others stay."""
    dk, dv = 4, 3
    r = _rng(23)
    S0 = r.standard_normal((1, 1, dv, dk))
    g = np.zeros((1, 1, 1, dk)); g[..., 2] = -60.0
    k = np.zeros((1, 1, 1, dk)); k[..., 0] = 1.0
    v = np.zeros((1, 1, 1, dv))
    _, fin, _ = run(k, k, v, g, np.zeros((1, 1, 1)), initial_state=S0)
    want = S0.copy(); want[..., 2] *= math.exp(-60.0)
    _close(fin, want, 1e-14, "per-channel gate acts on key channels")


# ---------------------------------------------------------------------------
# Sequence bookkeeping: snapshots, resume, packing, scale
# ---------------------------------------------------------------------------

def pin_snapshots_are_prefix_states(run):
    """A snapshot after n*stride tokens equals the final state of a run over
    that prefix alone ("Hybrid models ...", serving item 1), and resuming from
    it reproduces the rest of the run."""
    q, k, v, g, beta, S0 = _rand_problem(30, T=23, B=2)
    stride = 5
    out, fin, snaps = run(q, k, v, g, beta, initial_state=S0, snapshot_stride=stride)
    assert snaps.shape[1] == 23 // stride
    for s in range(snaps.shape[1]):
        n = (s + 1) * stride
        _, f_pre, _ = run(q[:, :n], k[:, :n], v[:, :n], g[:, :n], beta[:, :n], initial_state=S0)
        _close(snaps[:, s], f_pre, 0.0, f"snapshot {s}")
    n = 2 * stride
    o_rest, f_rest, _ = run(q[:, n:], k[:, n:], v[:, n:], g[:, n:], beta[:, n:], initial_state=snaps[:, 1])
    _close(o_rest, out[:, n:], 0.0, "resume outputs")
    _close(f_rest, fin, 0.0, "resume final state")


def pin_packed_equals_separate(run):
    """Packed sequences are independent: each one run alone gives the same."""
    lens = [7, 1, 13, 0, 5]
    T = sum(lens)
    q, k, v, g, beta, _ = _rand_problem(31, T=T, per_channel=True)
    S0 = _rng(32).standard_normal((len(lens), 2, 3, 5))
    cu = np.concatenate([[0], np.cumsum(lens)])
    out, fin, _ = run(q, k, v, g, beta, initial_state=S0, cu_seqlens=cu)
    for n, (a, b) in enumerate(zip(cu[:-1], cu[1:])):
        o1, f1, _ = run(q[:, a:b], k[:, a:b], v[:, a:b], g[:, a:b], beta[:, a:b], initial_state=S0[n:n + 1])
        _close(out[:, a:b], o1, 0.0, f"packed seq {n} outputs")
        _close(fin[n:n + 1], f1, 0.0, f"packed seq {n} state")


def pin_query_scale(run):
    """The query scale multiplies the read only: o = S_t (scale q_t)."""
    q, k, v, g, beta, S0 = _rand_problem(33, T=9)
    o1, f1, _ = run(q, k, v, g, beta, initial_state=S0)
    o2, f2, _ = run(q, k, v, g, beta, initial_state=S0, scale=0.25)
    _close(o2, 0.25 * o1, 1e-14, "scaled outputs")
    _close(f2, f1, 0.0, "scale leaves the state alone")


ALL_PINS = [v for k_, v in sorted(globals().items()) if k_.startswith("pin_")]
