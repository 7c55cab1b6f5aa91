"""Python binding of libgdn.so: argument marshalling for torch CUDA tensors.

Every step of the computation runs in the library's CUDA kernels; this module
only checks tensor placement/dtypes, allocates outputs and workspace with torch
when the caller does not pass them, and forwards pointers and the current CUDA
stream.  There is no CPU fallback: when ``libgdn.so`` is missing or cannot be
loaded, every call raises.

Names follow the C ABI in ``include/gdn.h``.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# GDN_LIBRARY may name another build of the library (the bounds-checked one, for tests).
LIB_PATH = os.environ.get("GDN_LIBRARY") or os.path.join(_PKG, "libgdn.so")

GDN_OK, GDN_ERR_INVALID_ARG, GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_ERR_CUDA, GDN_ERR_TIMEOUT, \
    GDN_ERR_INTERNAL = range(7)
GDN_F32, GDN_BF16 = 0, 1
GDN_GATE_HEAD, GDN_GATE_CHANNEL = 0, 1

GDN_DEV_OK, GDN_DEV_TIMEOUT_PREP, GDN_DEV_TIMEOUT_SCAN, GDN_DEV_BOUNDS = 0, 1, 2, 16

EXPORTED = ("gdn_chunk_workspace_size", "gdn_chunk_fwd", "gdn_chunk_status", "gdn_chunk_fwd_static",
            "gdn_chunk_status_static", "gdn_decode_step", "gdn_decode_multi", "gdn_state_select", "gdn_prerule",
            "gdn_decode_step_prerule", "gdn_status_string", "gdn_last_error", "gdn_profile_enable",
            "gdn_profile_read")


class GdnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int64),
                ("dk", ctypes.c_int64), ("dv", ctypes.c_int64), ("dtype", ctypes.c_int32),
                ("gate", ctypes.c_int32), ("scale", ctypes.c_float), ("hk", ctypes.c_int32)]


class GdnKernelTime(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int64), ("total_ms", ctypes.c_double)]


class GdnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


_lock = threading.Lock()
_lib = None


def load_library(path: str = LIB_PATH):
    """Load libgdn.so and declare its entry points.  Raises if it is missing."""
    global _lib
    with _lock:
        if _lib is not None and path == LIB_PATH:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with `python -m gated_delta_rule_64_b200.build`"
                               " (there is no CPU fallback)")
        lib = ctypes.CDLL(path)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        dp = ctypes.POINTER(GdnDesc)
        lib.gdn_chunk_workspace_size.argtypes = [dp, i32, ctypes.POINTER(sz)]
        lib.gdn_chunk_fwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, vp, sz, vp]
        lib.gdn_chunk_fwd_static.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, i64, vp, vp, vp, vp]
        lib.gdn_chunk_status.argtypes = [vp, vp, ctypes.POINTER(i32)]
        lib.gdn_chunk_status_static.argtypes = [vp, ctypes.POINTER(i32)]
        lib.gdn_decode_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.gdn_decode_multi.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, i32, vp, vp, vp]
        lib.gdn_state_select.argtypes = [dp, vp, vp, vp, vp]
        lib.gdn_prerule.argtypes = [dp, vp, vp, vp, vp, i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.gdn_decode_step_prerule.argtypes = [dp, vp, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp]
        lib.gdn_status_string.argtypes = [ctypes.c_int]
        lib.gdn_status_string.restype = ctypes.c_char_p
        lib.gdn_last_error.argtypes = []
        lib.gdn_last_error.restype = ctypes.c_char_p
        lib.gdn_profile_enable.argtypes = [ctypes.c_int]
        lib.gdn_profile_read.argtypes = [ctypes.POINTER(GdnKernelTime), i32, ctypes.POINTER(i32)]
        for name in ("gdn_chunk_workspace_size", "gdn_chunk_fwd", "gdn_chunk_status", "gdn_chunk_status_static",
                     "gdn_chunk_fwd_static", "gdn_decode_step",
                     "gdn_decode_multi", "gdn_state_select", "gdn_prerule", "gdn_decode_step_prerule",
                     "gdn_profile_enable", "gdn_profile_read"):
            getattr(lib, name).restype = ctypes.c_int
        if path == LIB_PATH:
            _lib = lib
        return lib


def _check(lib, st: int):
    if st != GDN_OK:
        msg = lib.gdn_last_error().decode() or lib.gdn_status_string(st).decode()
        raise GdnError(st, msg)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return GDN_F32
    if t.dtype == torch.bfloat16:
        return GDN_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be CUDA tensors (the library has no CPU path)")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def make_desc(B, T, H, dk, dv, dtype_code, per_channel, scale, hk=0) -> GdnDesc:
    """hk: query/key heads when fewer than the H value heads (0: H)."""
    return GdnDesc(B, T, H, dk, dv, dtype_code, GDN_GATE_CHANNEL if per_channel else GDN_GATE_HEAD,
                   float(scale), int(hk) if hk != H else 0)


def gdn_chunk_workspace_size(B, T, H, dk, dv, num_seqs, *, dtype=torch.bfloat16, per_channel=False,
                             hk=0) -> int:
    lib = load_library()
    d = make_desc(B, T, H, dk, dv, GDN_F32 if dtype == torch.float32 else GDN_BF16, per_channel, 1.0, hk)
    n = ctypes.c_size_t(0)
    _check(lib, lib.gdn_chunk_workspace_size(ctypes.byref(d), int(num_seqs), ctypes.byref(n)))
    return int(n.value)


def gdn_chunk_fwd(q, k, v, log_gate, beta, initial_state=None, cu_seqlens=None, *, scale=1.0,
                  snapshot_stride=0, out=None, final_state=True, snapshots=None, workspace=None,
                  stream=None):
    """Chunkwise prefill.  Shapes as in include/gdn.h:
    q, k (B,T,Hk,dk) with Hk dividing H (value head h reads query/key head h // (H // Hk)); v (B,T,H,dv); log_gate (B,T,H) or (B,T,H,dk); beta (B,T,H);
    initial_state (N,H,dv,dk) fp32 or None; cu_seqlens int32 (N+1) on the device or None.
    final_state: True to allocate, a tensor to fill (may be initial_state), or None.
    Returns (out, final_state, snapshots)."""
    lib = load_library()
    _need_cuda(q, k, v, log_gate, beta, initial_state, cu_seqlens)
    B, T, Hq, dk = q.shape
    H, dv = v.shape[-2], v.shape[-1]  # value heads; q and k may have fewer (Hq divides H)
    per_channel = log_gate.dim() == 4
    N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    dev = q.device
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    if final_state is True:
        final_state = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    elif final_state is False:
        final_state = None
    if snapshot_stride and snapshots is None:
        n_snap = T // snapshot_stride
        snapshots = torch.empty((B, n_snap, H, dv, dk), dtype=torch.float32, device=dev)
    d = make_desc(B, T, H, dk, dv, _dtype_code(q), per_channel, scale, Hq)
    if workspace is None:
        ws_bytes = gdn_chunk_workspace_size(B, T, H, dk, dv, N, dtype=q.dtype, per_channel=per_channel, hk=Hq)
        workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    _need_cuda(out, final_state, snapshots, workspace)
    st = lib.gdn_chunk_fwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_gate), _ptr(beta),
                           _ptr(initial_state), _ptr(cu_seqlens), int(N), int(snapshot_stride), _ptr(out),
                           _ptr(final_state), _ptr(snapshots), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    _check(lib, st)
    return out, final_state, snapshots


def gdn_chunk_status(workspace, stream=None):
    """Device status of the last gdn_chunk_fwd call that used `workspace` on `stream`
    (waits for the stream): (status, device_code); status GDN_OK, GDN_ERR_TIMEOUT
    or GDN_ERR_INTERNAL, device_code one of the GDN_DEV_* codes."""
    lib = load_library()
    _need_cuda(workspace)
    code = ctypes.c_int32(-1)
    st = lib.gdn_chunk_status(_ptr(workspace), _stream(stream), ctypes.byref(code))
    if st == GDN_ERR_CUDA or st == GDN_ERR_INVALID_ARG:
        _check(lib, st)
    return st, int(code.value)


def gdn_chunk_status_static(stream=None):
    """gdn_chunk_status for gdn_chunk_fwd_static (its built-in scratch on the current device)."""
    lib = load_library()
    code = ctypes.c_int32(-1)
    st = lib.gdn_chunk_status_static(_stream(stream), ctypes.byref(code))
    if st == GDN_ERR_CUDA or st == GDN_ERR_INVALID_ARG:
        _check(lib, st)
    return st, int(code.value)


def gdn_chunk_fwd_static(q, k, v, log_gate, beta, initial_state=None, cu_seqlens=None, *, scale=1.0,
                         snapshot_stride=0, out=None, final_state=True, snapshots=None, stream=None):
    """gdn_chunk_fwd for callers that cannot allocate device scratch: the library
    uses its built-in 64 MiB scratch array instead of a workspace (requests
    that need more are rejected).  This wrapper still allocates the outputs with
    torch when they are not passed; a caller that cannot allocate passes them."""
    lib = load_library()
    _need_cuda(q, k, v, log_gate, beta, initial_state, cu_seqlens)
    B, T, Hq, dk = q.shape
    H, dv = v.shape[-2], v.shape[-1]  # value heads; q and k may have fewer (Hq divides H)
    per_channel = log_gate.dim() == 4
    N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    dev = q.device
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    if final_state is True:
        final_state = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    elif final_state is False:
        final_state = None
    if snapshot_stride and snapshots is None:
        snapshots = torch.empty((B, T // snapshot_stride, H, dv, dk), dtype=torch.float32, device=dev)
    _need_cuda(out, final_state, snapshots)
    d = make_desc(B, T, H, dk, dv, _dtype_code(q), per_channel, scale, Hq)
    st = lib.gdn_chunk_fwd_static(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_gate), _ptr(beta),
                                  _ptr(initial_state), _ptr(cu_seqlens), int(N), int(snapshot_stride), _ptr(out),
                                  _ptr(final_state), _ptr(snapshots), _stream(stream))
    _check(lib, st)
    return out, final_state, snapshots


def gdn_decode_step(q, k, v, log_gate, beta, state, *, scale=1.0, out=None, stream=None):
    """One decode token per sequence; `state` (B,H,dv,dk) fp32 is updated in place.
    q, k (B,1,H,dk) or (B,H,dk); v (B,1,H,dv) or (B,H,dv); log_gate (B,[1,]H[,dk]); beta (B,[1,]H)."""
    lib = load_library()
    _need_cuda(q, k, v, log_gate, beta, state)
    B, H, dv, dk = state.shape
    per_channel = log_gate.dim() == q.dim()  # (.., H, dk) per channel, (.., H) per head
    if out is None:
        out = torch.empty((B, 1, H, dv), dtype=q.dtype, device=q.device)
    _need_cuda(out)
    d = make_desc(B, 1, H, dk, dv, _dtype_code(q), per_channel, scale, q.shape[-2])
    st = lib.gdn_decode_step(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_gate), _ptr(beta), _ptr(state),
                             _ptr(out), _stream(stream))
    _check(lib, st)
    return out


def gdn_decode_multi(q, k, v, log_gate, beta, state, *, n_tokens=None, commit=True, step_states=None, scale=1.0,
                     out=None, stream=None):
    """Up to T tokens per sequence in one pass over the state (speculative verify / multi-token decode).
    q, k (B,T,H,dk); v (B,T,H,dv); log_gate (B,T,H) or (B,T,H,dk); beta (B,T,H); state (B,H,dv,dk) fp32;
    n_tokens: int32 (B) on the device or None (all T); commit: write the state after n_tokens back;
    step_states: True to allocate, a (B,T,H,dv,dk) fp32 tensor, or None.  Returns (out, step_states)."""
    lib = load_library()
    _need_cuda(q, k, v, log_gate, beta, state)
    B, T, Hq, dk = q.shape
    H, dv = v.shape[-2], v.shape[-1]
    per_channel = log_gate.dim() == 4
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if step_states is True:
        step_states = torch.empty((B, T, H, dv, dk), dtype=torch.float32, device=q.device)
    _need_cuda(out)
    d = make_desc(B, T, H, dk, dv, _dtype_code(q), per_channel, scale, Hq)
    st = lib.gdn_decode_multi(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_gate), _ptr(beta),
                              _ptr(n_tokens), _ptr(state), 1 if commit else 0, _ptr(out), _ptr(step_states),
                              _stream(stream))
    _check(lib, st)
    return out, step_states


def gdn_prerule(x, a, b, conv_w, A_log, dt_bias, *, hk, dk, H, dv, cu_seqlens=None, conv_state_in=None,
                conv_state_out=None, stream=None):
    """Short convolution + SiLU, length-1 q/k and the gates from the raw projections.
    x (B,T,2*hk*dk+H*dv); a, b (B,T,H) in x's dtype; conv_w (C,K) fp32; A_log, dt_bias (H,) fp32;
    conv states (N,C,K-1) fp32 or None (conv_state_out may be conv_state_in).
    Returns (q (B,T,hk,dk), k, v (B,T,H,dv), log_gate (B,T,H), beta (B,T,H))."""
    lib = load_library()
    _need_cuda(x, a, b, conv_w, A_log, dt_bias, cu_seqlens, conv_state_in, conv_state_out)
    B, T, C = x.shape
    K = conv_w.shape[1]
    N = (cu_seqlens.numel() - 1) if cu_seqlens is not None else B
    dev = x.device
    q = torch.empty((B, T, hk, dk), dtype=x.dtype, device=dev)
    k = torch.empty((B, T, hk, dk), dtype=x.dtype, device=dev)
    v = torch.empty((B, T, H, dv), dtype=x.dtype, device=dev)
    g = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    beta = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    d = make_desc(B, T, H, dk, dv, _dtype_code(x), False, 1.0, hk)
    st = lib.gdn_prerule(ctypes.byref(d), _ptr(x), _ptr(a), _ptr(b), _ptr(conv_w), int(K), _ptr(A_log),
                         _ptr(dt_bias), _ptr(cu_seqlens), int(N), _ptr(conv_state_in), _ptr(conv_state_out),
                         _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _stream(stream))
    _check(lib, st)
    return q, k, v, g, beta


def gdn_decode_step_prerule(x, a, b, conv_w, A_log, dt_bias, conv_state, state, *, hk, dk, H, dv, scale=1.0,
                            out=None, stream=None):
    """One decode step from the raw projections: x (B,2*hk*dk+H*dv) (or (B,1,C)); a, b (B,H)
    (or (B,1,H)) in x's dtype; conv_w (C,K), A_log, dt_bias (H,) fp32; conv_state (B,C,K-1) fp32
    or None, updated in place; state (B,H,dv,dk) fp32, updated in place.  Returns out (B,H,dv)."""
    lib = load_library()
    _need_cuda(x, a, b, conv_w, A_log, dt_bias, conv_state, state)
    B = x.shape[0]
    K = conv_w.shape[1]
    if out is None:
        out = torch.empty((B, H, dv), dtype=x.dtype, device=x.device)
    d = make_desc(B, 1, H, dk, dv, _dtype_code(x), False, scale, hk)
    _check(lib, lib.gdn_decode_step_prerule(ctypes.byref(d), _ptr(x), _ptr(a), _ptr(b), _ptr(conv_w), int(K),
                                            _ptr(A_log), _ptr(dt_bias), _ptr(conv_state), _ptr(state), _ptr(out),
                                            _stream(stream)))
    return out


def gdn_state_select(step_states, accept, state, *, stream=None):
    """state[b] = step_states[b, accept[b] - 1] where accept[b] > 0 (int32 device tensor)."""
    lib = load_library()
    _need_cuda(step_states, accept, state)
    B, T, H, dv, dk = step_states.shape
    d = make_desc(B, T, H, dk, dv, GDN_F32, False, 1.0)
    _check(lib, lib.gdn_state_select(ctypes.byref(d), _ptr(step_states), _ptr(accept), _ptr(state),
                                     _stream(stream)))
    return state


def profile_enable(on: bool = True):
    lib = load_library()
    _check(lib, lib.gdn_profile_enable(1 if on else 0))


def profile_read() -> dict:
    """{kernel name: (launches, total ms)} since the last read (waits for the events)."""
    lib = load_library()
    cap = 64
    arr = (GdnKernelTime * cap)()
    cnt = ctypes.c_int32(0)
    _check(lib, lib.gdn_profile_read(arr, cap, ctypes.byref(cnt)))
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(min(cap, cnt.value))}
