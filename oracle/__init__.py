"""fp64 CPU oracle of the gated delta rule -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does, and this
package imports nothing from it.

The arithmetic lives in ``gdn_oracle.c`` (a plain token loop in double
precision, see that file's header for the sources); this module only builds it
with gcc, converts tensors to fp64 arrays and unpacks the results.

Every input is upcast exactly (bf16 and fp32 values are representable in fp64),
so the oracle sees the same numbers the GPU path rounds its inputs to.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH) -> str:
    """Compile the oracle's C source into a shared library with gcc (IEEE fp64, no fast-math)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
                        src, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, out)
    return out


def bind(path: str):
    """Load a compiled oracle library and declare its entry point."""
    lib = ctypes.CDLL(path)
    f = lib.oracle_gdn_forward
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int64, _i64p, _i64p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                  _dp, _dp, _dp, _dp, _dp, _dp,
                  ctypes.c_int, ctypes.c_int, ctypes.c_double,
                  ctypes.c_int64, ctypes.c_int64,
                  _dp, _dp, _dp, ctypes.c_int]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = bind(build())
    return _lib


def host_threads() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _f64(x) -> np.ndarray:
    """Exact upcast of a torch tensor (any float dtype, incl. bf16) or array to fp64."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return np.ascontiguousarray(x.detach().to("cpu", torch.float64).numpy())
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def gated_delta_rule(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *,
                     per_channel: bool | None = None, additive: bool = False, scale: float = 1.0,
                     snapshot_stride: int = 0, n_threads: int | None = None, lib=None):
    """Run the recurrence token by token in fp64.

    Shapes (the library's layout):
      q, k: (B, T, H, dk); v: (B, T, H, dv)
      g:    (B, T, H) for one gate per head, or (B, T, H, dk) per channel (KDA)
            -- the gate as a logarithm, g = log(alpha)
      beta: (B, T, H)
      initial_state: (N, H, dv, dk) or None for zeros
      cu_seqlens: None (N = B sequences of length T) or N+1 packed offsets into
            the flattened B*T token rows (then B must be 1)
    Returns (out (B,T,H,dv), final_state (N,H,dv,dk), snapshots or None) as
    float64 numpy arrays; snapshots is (N, max_n floor(len_n/stride), H, dv, dk),
    zero where a sequence has fewer snapshots.  `lib` selects another build of
    the same C source (the tests use it to check that the pins reject planted
    mistakes).
    """
    q, k, v, g, beta = (_f64(t) for t in (q, k, v, g, beta))
    h0 = _f64(initial_state)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if per_channel is None:
        per_channel = g.ndim == 4
    rows = B * T
    if cu_seqlens is None:
        starts = np.arange(B, dtype=np.int64) * T
        lens = np.full(B, T, dtype=np.int64)
    else:
        cs = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64)
        if B != 1:
            raise ValueError("packed sequences need B == 1")
        starts = np.ascontiguousarray(cs[:-1])
        lens = np.ascontiguousarray(cs[1:] - cs[:-1])
        if lens.size and (lens.min() < 0 or cs[-1] > rows or cs[0] < 0):
            raise ValueError("bad cu_seqlens")
    starts = np.ascontiguousarray(starts, dtype=np.int64)
    lens = np.ascontiguousarray(lens, dtype=np.int64)
    N = lens.size
    if h0 is not None and h0.shape != (N, H, dv, dk):
        raise ValueError(f"initial_state must be {(N, H, dv, dk)}, got {h0.shape}")
    out = np.zeros((B, T, H, dv), dtype=np.float64)
    final = np.zeros((N, H, dv, dk), dtype=np.float64)
    n_snap = int(lens.max() // snapshot_stride) if (snapshot_stride and N) else 0
    snaps = np.zeros((N, n_snap, H, dv, dk), dtype=np.float64)
    rc = (lib or _load()).oracle_gdn_forward(
        N, starts.ctypes.data_as(_i64p), lens.ctypes.data_as(_i64p), H, dk, dv,
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(h0),
        int(bool(per_channel)), int(bool(additive)), float(scale),
        int(snapshot_stride), n_snap, _ptr(out), _ptr(final), _ptr(snaps) if n_snap else None,
        int(n_threads or host_threads()))
    if rc != 0:
        raise ValueError(f"oracle rejected its arguments (rc={rc})")
    return out, final, (snaps if snapshot_stride else None)
