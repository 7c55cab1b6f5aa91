"""gdn_chunk_fwd_static: the prefill entry point that allocates nothing.

It serves callers that cannot allocate device memory -- a serving loop whose
allocator owns a fixed device budget, a real-time path that must not take the
synchronisation an allocation can cause, a plugin handed pointers but no
allocator.  Its scratch is a fixed array built into the library, shared by
every call.

Checked here, through the C ABI: two calls in a row (different sizes and
precisions, so the second one runs over whatever the first left in the shared
array) each match gdn_chunk_fwd with a caller-provided workspace on the same
inputs, within the parity tolerances of the other GPU tests; and a request
larger than the built-in scratch is refused before anything runs.

The file name makes pytest collect it last, after every other test.
"""
import ctypes

import pytest
import torch

from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import Workload, make_inputs
from tests.gpu_util import rel_l2, tolerances, to_dev

pytestmark = pytest.mark.gpu


def _call_static(lib, dx, out, fin):
    B, T, H, dk = dx.q.shape
    dv = dx.v.shape[-1]
    d = gdn.make_desc(B, T, H, dk, dv, gdn._dtype_code(dx.q), dx.g.dim() == 4, 1.0)
    st = lib.gdn_chunk_fwd_static(ctypes.byref(d), gdn._ptr(dx.q), gdn._ptr(dx.k), gdn._ptr(dx.v), gdn._ptr(dx.g),
                                  gdn._ptr(dx.beta), gdn._ptr(dx.h0), None, B, 0, gdn._ptr(out), gdn._ptr(fin), None,
                                  gdn._stream(None))
    assert st == gdn.GDN_OK, lib.gdn_last_error().decode()


def test_static_scratch_matches_workspace_path_on_two_calls():
    lib = gdn.load_library()
    cases = [Workload("no-alloc a", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=41),
             Workload("no-alloc b", B=3, T=200, H=2, dk=64, dv=64, dtype="f32", h0_std=0.1, seed=42)]
    for w in cases:
        x = make_inputs(w)
        dx = to_dev(x)
        B, T, H, dk = dx.q.shape
        out = torch.empty((B, T, H, w.dv), dtype=dx.q.dtype, device="cuda")
        fin = torch.empty((B, H, w.dv, dk), dtype=torch.float32, device="cuda")
        _call_static(lib, dx, out, fin)
        o_ref, f_ref, _ = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0)
        torch.cuda.synchronize()
        tol_o, tol_s = tolerances(dx.q.dtype)
        assert rel_l2(out, o_ref.cpu().double().numpy()) <= tol_o
        assert rel_l2(fin, f_ref.cpu().double().numpy()) <= tol_s


def test_static_scratch_rejects_oversized_requests():
    lib = gdn.load_library()
    d = gdn.make_desc(4, 40000, 16, 128, 128, gdn.GDN_BF16, False, 1.0)
    fake = [ctypes.c_void_p(1 << 40) for _ in range(7)]
    st = lib.gdn_chunk_fwd_static(ctypes.byref(d), *fake[:5], None, None, 4, 0, fake[5], fake[6], None, None)
    assert st == gdn.GDN_ERR_WORKSPACE
    assert "scratch" in lib.gdn_last_error().decode()
