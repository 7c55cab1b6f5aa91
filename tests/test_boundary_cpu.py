"""The C-ABI library on the host: it loads, exports every declared entry point,
and rejects bad arguments before launching anything (no GPU needed: every case
here fails validation, so no CUDA call is reached)."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_64_b200 import gdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_64_b200 import build
    build.build()
    return gdn.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gdn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gdn_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(gdn.EXPORTED), names
    for n in names:
        assert hasattr(lib, n), n


def test_struct_layout_matches_header():
    assert ctypes.sizeof(gdn.GdnDesc) == 56


def _desc(B=2, T=130, H=3, dk=128, dv=128, dtype=gdn.GDN_BF16, gate=gdn.GDN_GATE_HEAD, scale=1.0):
    return gdn.GdnDesc(B, T, H, dk, dv, dtype, gate, scale, 0)


A = 1 << 40  # fake, 256-byte aligned "device" addresses; never dereferenced


def _addr(i, off=0):
    return ctypes.c_void_p(A + i * (1 << 32) + off)


def _fwd(lib, d, *, q=0, k=1, v=2, g=3, beta=4, h0=None, cu=None, n=0, snap=0, out=5, fin=None, snaps=None,
         ws=7, ws_bytes=1 << 40, off=None):
    off = off or {}
    p = lambda i, name: None if i is None else _addr(i, off.get(name, 0))
    return lib.gdn_chunk_fwd(ctypes.byref(d), p(q, "q"), p(k, "k"), p(v, "v"), p(g, "g"), p(beta, "beta"),
                             p(h0, "h0"), p(cu, "cu"), n, snap, p(out, "out"), p(fin, "fin"), p(snaps, "snaps"),
                             p(ws, "ws"), ws_bytes, None)


def test_workspace_size(lib):
    # 2 sequences of 130 tokens: at most 260/64 + 2 = 6 chunks x 3 heads
    def size(**kw):
        n = ctypes.c_size_t()
        d = _desc(**kw)
        assert lib.gdn_chunk_workspace_size(ctypes.byref(d), 2, ctypes.byref(n)) == gdn.GDN_OK
        return n.value
    simt = 4 * 64 * (128 + 128 + 64 + 1)          # fp32 W, U, P and gate per chunk-head
    assert 6 * 3 * simt <= size(dtype=gdn.GDN_F32) < 6 * 3 * simt + 4096
    tc = 32768 + 64 * 128 * 2 + 64 * 128 + 64 * 128 + 1024  # W^T and Qs rows, K~, P rows, -T'' rows, factors
    assert 6 * 3 * tc <= size() < 6 * 3 * tc + 4096
    # the per-channel gate uses the same block
    assert 6 * 3 * tc <= size(gate=gdn.GDN_GATE_CHANNEL) < 6 * 3 * tc + 4096
    assert size(dtype=gdn.GDN_F32, gate=gdn.GDN_GATE_CHANNEL) > size(dtype=gdn.GDN_F32)
    d = _desc()
    assert lib.gdn_chunk_workspace_size(ctypes.byref(d), 2, None) == gdn.GDN_ERR_INVALID_ARG


@pytest.mark.parametrize("field,value,status", [
    ("dk", 96, gdn.GDN_ERR_UNSUPPORTED),
    ("dv", 32, gdn.GDN_ERR_UNSUPPORTED),
    ("H", 0, gdn.GDN_ERR_INVALID_ARG),
    ("T", -1, gdn.GDN_ERR_INVALID_ARG),
    ("dtype", 7, gdn.GDN_ERR_INVALID_ARG),
    ("gate", 3, gdn.GDN_ERR_INVALID_ARG),
    ("hk", 2, gdn.GDN_ERR_INVALID_ARG),   # H = 3: not a divisor
    ("hk", -1, gdn.GDN_ERR_INVALID_ARG),
    ("hk", 6, gdn.GDN_ERR_INVALID_ARG),
    ("scale", float("nan"), gdn.GDN_ERR_INVALID_ARG),
])
def test_bad_descriptor(lib, field, value, status):
    d = _desc()
    setattr(d, field, value)
    assert _fwd(lib, d) == status
    assert lib.gdn_last_error().decode()


def test_null_descriptor(lib):
    assert lib.gdn_chunk_fwd(None, *([None] * 7), 0, 0, None, None, None, None, 0, None) == gdn.GDN_ERR_INVALID_ARG


@pytest.mark.parametrize("name,off", [("q", 8), ("k", 8), ("v", 8), ("out", 8), ("g", 2), ("beta", 1),
                                      ("h0", 8)])
def test_misaligned_pointer(lib, name, off):
    kw = {"h0": 10} if name == "h0" else {}
    assert _fwd(lib, _desc(), off={name: off}, **kw) == gdn.GDN_ERR_INVALID_ARG
    assert "aligned" in lib.gdn_last_error().decode()


def test_gates_need_only_4_byte_alignment(lib):
    # passes validation (so it reaches the launch, which fails without a GPU)
    st = _fwd(lib, _desc(), off={"g": 4, "beta": 8})
    assert st in (gdn.GDN_OK, gdn.GDN_ERR_CUDA), st


def test_per_channel_gate_alignment(lib):
    d = _desc(gate=gdn.GDN_GATE_CHANNEL)
    assert _fwd(lib, d, off={"g": 4}) == gdn.GDN_ERR_INVALID_ARG
    assert "16-byte" in lib.gdn_last_error().decode()
    st = _fwd(lib, _desc(gate=gdn.GDN_GATE_CHANNEL), off={"g": 16, "beta": 4})
    assert st in (gdn.GDN_OK, gdn.GDN_ERR_CUDA), st


@pytest.mark.parametrize("name", ["q", "k", "v", "g", "beta", "out"])
def test_null_required_pointer(lib, name):
    kw = {name: None}
    assert _fwd(lib, _desc(), **kw) == gdn.GDN_ERR_INVALID_ARG


def test_out_overlapping_input(lib):
    # out starts inside v
    assert _fwd(lib, _desc(), out=2, off={"out": 256}) == gdn.GDN_ERR_INVALID_ARG
    assert "overlap" in lib.gdn_last_error().decode()


def test_workspace_checks(lib):
    assert _fwd(lib, _desc(), ws=None) == gdn.GDN_ERR_WORKSPACE
    assert _fwd(lib, _desc(), ws_bytes=1024) == gdn.GDN_ERR_WORKSPACE
    assert _fwd(lib, _desc(), off={"ws": 16}) == gdn.GDN_ERR_WORKSPACE


def test_snapshot_rules(lib):
    d = _desc(T=512)
    assert _fwd(lib, d, snap=100, snaps=8) == gdn.GDN_ERR_INVALID_ARG        # not a multiple of 64
    assert _fwd(lib, d, snap=-64, snaps=8) == gdn.GDN_ERR_INVALID_ARG
    assert _fwd(lib, d, snap=128, snaps=None) == gdn.GDN_ERR_INVALID_ARG     # buffer required
    dp = _desc(B=1, T=512)
    assert _fwd(lib, dp, cu=9, n=3, snap=128, snaps=8) == gdn.GDN_ERR_UNSUPPORTED


def test_packed_rules(lib):
    assert _fwd(lib, _desc(B=2), cu=9, n=2) == gdn.GDN_ERR_INVALID_ARG       # packing needs B == 1
    assert _fwd(lib, _desc(B=1), cu=9, n=-1) == gdn.GDN_ERR_INVALID_ARG
    assert _fwd(lib, _desc(B=1), cu=9, n=2, off={"cu": 2}) == gdn.GDN_ERR_INVALID_ARG


def test_final_state_partial_overlap(lib):
    assert _fwd(lib, _desc(), h0=10, fin=10, off={"fin": 256}) == gdn.GDN_ERR_INVALID_ARG


def test_decode_validation(lib):
    # argument order: q, k, v, log_gate, beta, state, out
    d = _desc(B=4, T=2)
    p = [_addr(i) for i in range(7)]
    assert lib.gdn_decode_step(ctypes.byref(d), *p, None) == gdn.GDN_ERR_INVALID_ARG   # T must be 1
    d = _desc(B=4, T=1)
    q = list(p)
    q[5] = None  # state
    assert lib.gdn_decode_step(ctypes.byref(d), *q, None) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[6] = _addr(5, 64)  # out inside the state
    assert lib.gdn_decode_step(ctypes.byref(d), *q, None) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[5] = _addr(0, 256)  # state overlapping q
    assert lib.gdn_decode_step(ctypes.byref(d), *q, None) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[0] = _addr(0, 4)  # misaligned q
    assert lib.gdn_decode_step(ctypes.byref(d), *q, None) == gdn.GDN_ERR_INVALID_ARG
    d = _desc(B=4, T=1, dk=32)
    assert lib.gdn_decode_step(ctypes.byref(d), *p, None) == gdn.GDN_ERR_UNSUPPORTED


def _multi(lib, d, p, commit=1):
    # argument order: q, k, v, log_gate, beta, n_tokens, state, commit, out, step_states
    return lib.gdn_decode_multi(ctypes.byref(d), p[0], p[1], p[2], p[3], p[4], p[5], p[6], commit, p[7], p[8], None)


def test_decode_multi_validation(lib):
    p = [_addr(i) for i in range(9)]
    for T in (0, 65):  # 1 .. 64 token slots
        assert _multi(lib, _desc(B=4, T=T), p) == gdn.GDN_ERR_INVALID_ARG
    d = _desc(B=4, T=8)
    assert _multi(lib, d, p, commit=2) == gdn.GDN_ERR_INVALID_ARG
    for i, bad in ((6, None), (0, None), (7, None)):  # state, q, out are required
        q = list(p)
        q[i] = bad
        assert _multi(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[8] = _addr(6, 4096)  # step_states inside the state
    assert _multi(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    assert "overlap" in lib.gdn_last_error().decode()
    q = list(p)
    q[7] = _addr(8, 16)  # out inside step_states
    assert _multi(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[5] = _addr(5, 2)  # misaligned n_tokens
    assert _multi(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[8] = _addr(8, 8)  # misaligned step_states
    assert _multi(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    # optional pointers may be NULL: validation passes (the launch then needs a GPU)
    q = list(p)
    q[5] = None
    q[8] = None
    assert _multi(lib, d, q) in (gdn.GDN_OK, gdn.GDN_ERR_CUDA)
    assert _multi(lib, _desc(B=0, T=8), p) == gdn.GDN_OK


def test_state_select_validation(lib):
    d = _desc(B=4, T=8)
    ss, acc, st = _addr(0), _addr(1), _addr(2)
    sel = lambda d, a, b, c: lib.gdn_state_select(ctypes.byref(d), a, b, c, None)
    assert sel(_desc(B=4, T=0), ss, acc, st) == gdn.GDN_ERR_INVALID_ARG
    assert sel(d, None, acc, st) == gdn.GDN_ERR_INVALID_ARG
    assert sel(d, ss, _addr(1, 2), st) == gdn.GDN_ERR_INVALID_ARG
    assert sel(d, ss, acc, _addr(0, 1024)) == gdn.GDN_ERR_INVALID_ARG  # state inside step_states
    assert sel(d, ss, acc, st) in (gdn.GDN_OK, gdn.GDN_ERR_CUDA)


def _prerule(lib, d, p, K=4, cu=None, n=0):
    # argument order: x, a, b, conv_w, A_log, dt_bias, state_in, state_out, q, k, v, log_gate, beta
    return lib.gdn_prerule(ctypes.byref(d), p[0], p[1], p[2], p[3], K, p[4], p[5], cu, n, p[6], p[7], p[8], p[9],
                           p[10], p[11], p[12], None)


def test_prerule_validation(lib):
    p = [_addr(i) for i in range(13)]
    d = _desc(B=2, T=16, H=4, dk=64, dv=64)
    assert _prerule(lib, d, p, K=0) == gdn.GDN_ERR_UNSUPPORTED
    assert _prerule(lib, d, p, K=5) == gdn.GDN_ERR_UNSUPPORTED
    assert _prerule(lib, _desc(B=2, T=16, H=4, dk=64, dv=64, gate=gdn.GDN_GATE_CHANNEL), p) == gdn.GDN_ERR_UNSUPPORTED
    assert _prerule(lib, d, p, cu=_addr(13), n=2) == gdn.GDN_ERR_INVALID_ARG  # packed needs B == 1
    q = list(p)
    q[8] = None
    assert _prerule(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[0] = _addr(0, 8)  # x not 16-byte aligned
    assert _prerule(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[9] = _addr(0, 64)  # k inside x
    assert _prerule(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[7] = _addr(6, 16)  # state_out partly over state_in
    assert _prerule(lib, d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[7] = q[6]  # in place is fine
    assert _prerule(lib, d, q) in (gdn.GDN_OK, gdn.GDN_ERR_CUDA)


def test_fused_decode_validation(lib):
    """gdn_decode_step_prerule: T == 1, the per-head gate, K in 1..4, required pointers,
    alignment and overlap checks, before any launch."""
    call = lambda d, p, K=4: lib.gdn_decode_step_prerule(ctypes.byref(d), p[0], p[1], p[2], p[3], K, p[4], p[5],
                                                         p[6], p[7], p[8], None)
    p = [_addr(i) for i in range(9)]
    d = _desc(B=2, T=1, H=4, dk=64, dv=64)
    assert call(_desc(B=2, T=2, H=4, dk=64, dv=64), p) == gdn.GDN_ERR_INVALID_ARG
    assert call(_desc(B=2, T=1, H=4, dk=64, dv=64, gate=gdn.GDN_GATE_CHANNEL), p) == gdn.GDN_ERR_UNSUPPORTED
    assert call(d, p, K=0) == gdn.GDN_ERR_UNSUPPORTED and call(d, p, K=5) == gdn.GDN_ERR_UNSUPPORTED
    for i in (0, 1, 2, 3, 4, 5, 7, 8):  # every pointer but conv_state is required
        q = list(p)
        q[i] = None
        assert call(d, q) == gdn.GDN_ERR_INVALID_ARG, i
    q = list(p)
    q[7] = _addr(7, 8)  # state not 16-byte aligned
    assert call(d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[8] = _addr(0, 64)  # out inside x
    assert call(d, q) == gdn.GDN_ERR_INVALID_ARG
    q = list(p)
    q[6] = _addr(7, 256)  # conv_state over the state
    assert call(d, q) == gdn.GDN_ERR_INVALID_ARG
    assert call(_desc(B=0, T=1, H=4, dk=64, dv=64), p) == gdn.GDN_OK


def test_status_strings(lib):
    for s in range(7):
        assert lib.gdn_status_string(s)
    assert lib.gdn_status_string(99) == b"unknown status"


def test_profile_api_without_launches(lib):
    assert lib.gdn_profile_enable(1) == gdn.GDN_OK
    cnt = ctypes.c_int32(-1)
    assert lib.gdn_profile_read(None, 0, ctypes.byref(cnt)) == gdn.GDN_OK
    assert cnt.value == 0
    assert lib.gdn_profile_enable(0) == gdn.GDN_OK


def test_python_binding_refuses_cpu_tensors(lib):
    import torch
    x = torch.zeros(1, 64, 1, 64)
    with pytest.raises(ValueError, match="CUDA"):
        gdn.gdn_chunk_fwd(x, x, x, torch.zeros(1, 64, 1), torch.zeros(1, 64, 1))


def _split_policy(N, H, nch, sms=148):
    """Segments per sequence the split scan picks, restated from the host code's cost
    model (chunk steps of one block): with gates that forget, waves of pass 1 x chunks
    per segment plus a short pass 2 and the launches; chosen as long as gates that
    keep the state alive (transition maps in pass 1, whole segments in pass 2) cost
    at most 1.3 times the unsplit scan."""
    waves = lambda ctas: -(-ctas // sms)
    best = (1, nch)
    if nch < 64:
        return best
    unsplit = waves(N * H) * nch
    best_cost = 0.95 * unsplit
    for G in range(2, 129):
        seg = -(-nch // G)
        if seg < 32:
            break
        Gr = -(-nch // seg)
        if Gr < 2:
            continue
        comb = 4.0 if Gr >= 3 else 0.0
        fast = waves(N * H * Gr) * seg + min(seg, 16.0) + 4.0 + comb + 0.5 * (Gr - 2)
        slow = waves(N * H * (2 * Gr - 2)) * seg + waves(N * H * (Gr - 1)) * seg + 4.0 + comb + 4.0 * (Gr - 2)
        if fast < best_cost and slow <= 1.3 * unsplit:
            best, best_cost = (Gr, seg), fast
    return best


def test_split_scan_workspace(lib):
    """Long fixed-length sequences on few (sequence, head) pairs get the split scan and
    its per-segment state maps in the workspace; short or many sequences do not.
    (Without a GPU the library plans for 148 multiprocessors.)"""
    def size(**kw):
        n = ctypes.c_size_t()
        d = _desc(**kw)
        assert lib.gdn_chunk_workspace_size(ctypes.byref(d), kw.get("B", 2), ctypes.byref(n)) == gdn.GDN_OK
        return n.value
    blk = 32768 + 64 * 128 * 2 + 64 * 128 + 64 * 128 + 1024  # the tensor-core block of a chunk-head
    up = lambda x: -(-x // 256) * 256
    state = 128 * 128 * 4

    def expect(N, H, nch, G):
        # status slot, chunk table, blocks, then (split) the segment states and records
        head = 256 + up(4 * (2 * N + 1))
        fixed = head + N * nch * H * blk + (up(N * G * 3 * H * state + 4 * 2 * N * G * H) if G >= 2 else 0)
        packed = head + (N * nch + N) * H * blk
        return max(fixed, packed)
    # one sequence of 262144 tokens, 16 heads: 4096 chunks, split so one wave holds pass 1
    G, seg = _split_policy(1, 16, 4096)
    assert G >= 3 and (G - 1) * seg < 4096 <= G * seg and 16 * G <= 148
    got = size(B=1, T=262144, H=16)
    assert expect(1, 16, 4096, G) <= got < expect(1, 16, 4096, G) + 1024
    # the prefill workload (64 (sequence, head) pairs of 64 chunks): two segments
    assert _split_policy(4, 16, 64) == (2, 32)
    got = size(B=4, T=4096, H=16)
    assert expect(4, 16, 64, 2) <= got < expect(4, 16, 64, 2) + 1024
    # many pairs: no split
    assert _split_policy(64, 16, 64) == (1, 64)
