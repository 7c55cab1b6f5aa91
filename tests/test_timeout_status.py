"""The device status word of the chunked prefill: a bounded device-side wait that
runs out is reported to the caller as GDN_ERR_TIMEOUT, and the GPU keeps working.

No kernel of the library is made to fail.  A test-only kernel (tests/csrc/
stuck_wait.cu, built here into its own small library) waits through the
library's bounded wait on an mbarrier that nobody arrives at, with a poll limit
of a few thousand, and records the scan's timeout code in a workspace's status
word with the library's own flag_error; nothing is in flight when it gives up, so
it ends by itself.  gdn_chunk_status then reads that word through the C ABI."""
import ctypes
import os
import subprocess

import pytest
import torch

from gated_delta_rule_64_b200 import build as gdn_build
from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import Workload, make_inputs
from tests.gpu_util import check_against_oracle, to_dev

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "stuck_wait.cu")
LIB = os.path.join(HERE, "_build", "libgdn_stuck.so")


def _stuck_lib():
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(os.path.getmtime(p) for p in gdn_build.deps() + [SRC]):
        os.makedirs(os.path.dirname(LIB), exist_ok=True)
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([gdn_build.nvcc(), *gdn_build.ARCH, "-O2", "-std=c++17", "-DGDN_CHECKED", "-Xcompiler",
                        "-fPIC", "-shared", "-I", gdn_build.INCLUDE, "-I", gdn_build.CSRC, SRC, "-o", tmp], check=True)
        os.replace(tmp, LIB)
    lib = ctypes.CDLL(LIB)
    lib.gdn_test_stuck_wait.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p, ctypes.c_void_p]
    lib.gdn_test_stuck_wait.restype = ctypes.c_int
    lib.gdn_test_bounds.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.c_void_p]
    lib.gdn_test_bounds.restype = ctypes.c_int
    return lib


W = Workload("status", B=2, T=200, H=2, dk=128, dv=128, dtype="bf16", h0_std=0.05, seed=61)


def _run(x, ws):
    dx = to_dev(x)
    out, fin, _ = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0, workspace=ws)
    return out, fin


def test_timeout_is_reported_and_the_gpu_keeps_working():
    lib = _stuck_lib()
    x = make_inputs(W)
    ws = torch.empty(gdn.gdn_chunk_workspace_size(2, 200, 2, 128, 128, 2), dtype=torch.uint8, device="cuda")
    _run(x, ws)
    assert gdn.gdn_chunk_status(ws) == (gdn.GDN_OK, gdn.GDN_DEV_OK)

    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    assert lib.gdn_test_stuck_wait(ctypes.c_void_p(ws.data_ptr()), 4096, ctypes.c_void_p(gave_up.data_ptr()),
                                   ctypes.c_void_p(stream.cuda_stream)) == 0
    st, code = gdn.gdn_chunk_status(ws)
    assert st == gdn.GDN_ERR_TIMEOUT and code == gdn.GDN_DEV_TIMEOUT_SCAN
    assert int(gave_up.item()) == 1
    assert "gave up" in gdn.load_library().gdn_last_error().decode()

    # the context still works: the next call clears the word and computes correctly
    out, fin = _run(x, ws)
    assert gdn.gdn_chunk_status(ws) == (gdn.GDN_OK, gdn.GDN_DEV_OK)
    check_against_oracle(x, out, fin)


def test_status_of_the_static_entry_point():
    x = make_inputs(W.replace(seed=62))
    dx = to_dev(x)
    out, fin, _ = gdn.gdn_chunk_fwd_static(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0)
    assert gdn.gdn_chunk_status_static() == (gdn.GDN_OK, gdn.GDN_DEV_OK)
    check_against_oracle(x, out, fin)


def test_bounds_code_is_reported():
    """The range check of the bounds-checked build (in_bounds, as its kernels use it)
    fails on an index one past its size: the guarded store is skipped, GDN_DEV_BOUNDS
    is recorded and gdn_chunk_status returns GDN_ERR_INTERNAL."""
    lib = _stuck_lib()
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    dst = torch.zeros(9, dtype=torch.float32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    assert lib.gdn_test_bounds(p(ws), 3, 8, p(dst), stream) == 0
    assert gdn.gdn_chunk_status(ws) == (gdn.GDN_OK, gdn.GDN_DEV_OK)
    assert lib.gdn_test_bounds(p(ws), 8, 8, p(dst), stream) == 0
    assert gdn.gdn_chunk_status(ws) == (gdn.GDN_ERR_INTERNAL, gdn.GDN_DEV_BOUNDS)
    assert dst.cpu().tolist() == [0, 0, 0, 1, 0, 0, 0, 0, 0]
