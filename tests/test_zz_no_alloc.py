"""gdn_chunk_fwd_static: the prefill entry point that allocates nothing.

It serves callers that cannot allocate device memory -- a serving loop whose
allocator owns a fixed device budget, a real-time path that must not take the
synchronisation an allocation can cause, a plugin handed pointers but no
allocator.  Its scratch is a fixed array built into the library, shared by
every call.

Checked here, through the C ABI:
  * calls in a row (different sizes, precisions, a packed batch and a long
    sequence that takes the split scan, each running over whatever the call
    before left in the shared array) give exactly gdn_chunk_fwd's results with a
    caller-provided workspace -- bit for bit, since the same kernels run;
  * a request larger than the built-in scratch is refused before anything runs;
  * in a fresh process, a first static call leaves the device memory in use
    unchanged (the array itself is counted before: under CUDA's lazy module
    loading it appears when the library first looks up its address).

The file name makes pytest collect it last, after every other test.
"""
import ctypes
import os
import subprocess
import sys

import pytest
import torch

from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import Workload, make_inputs
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _call_static(lib, dx, out, fin, snaps=None, stride=0):
    B, T, H, dk = dx.q.shape
    dv = dx.v.shape[-1]
    N = dx.cu_seqlens.numel() - 1 if dx.cu_seqlens is not None else B
    d = gdn.make_desc(B, T, H, dk, dv, gdn._dtype_code(dx.q), dx.g.dim() == 4, 1.0)
    st = lib.gdn_chunk_fwd_static(ctypes.byref(d), gdn._ptr(dx.q), gdn._ptr(dx.k), gdn._ptr(dx.v), gdn._ptr(dx.g),
                                  gdn._ptr(dx.beta), gdn._ptr(dx.h0), gdn._ptr(dx.cu_seqlens), N, stride,
                                  gdn._ptr(out), gdn._ptr(fin), gdn._ptr(snaps), gdn._stream(None))
    assert st == gdn.GDN_OK, lib.gdn_last_error().decode()


CASES = [
    (Workload("no-alloc large", B=1, T=16384, H=2, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=40), None, 0),
    (Workload("no-alloc a", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=41), None, 0),
    (Workload("no-alloc b", B=3, T=200, H=2, dk=64, dv=64, dtype="f32", h0_std=0.1, seed=42), None, 0),
    (Workload("no-alloc packed", B=1, T=0, H=3, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=43),
     [70, 1, 300, 0, 129], 0),
    (Workload("no-alloc split", B=1, T=8192, H=2, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=44), None, 1024),
]


def test_static_scratch_matches_workspace_path_bit_for_bit():
    lib = gdn.load_library()
    for w, lengths, stride in CASES:
        x = make_inputs(w, lengths=lengths)
        dx = to_dev(x)
        B, T, H, dk = dx.q.shape
        N = x.n_seqs
        out = torch.empty((B, T, H, w.dv), dtype=dx.q.dtype, device="cuda")
        fin = torch.empty((N, H, w.dv, dk), dtype=torch.float32, device="cuda")
        snaps = torch.empty((N, T // stride, H, w.dv, dk), dtype=torch.float32, device="cuda") if stride else None
        _call_static(lib, dx, out, fin, snaps, stride)
        assert gdn.gdn_chunk_status_static() == (gdn.GDN_OK, gdn.GDN_DEV_OK)
        o_ref, f_ref, s_ref = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0, dx.cu_seqlens,
                                                snapshot_stride=stride)
        torch.cuda.synchronize()
        assert torch.equal(out, o_ref), w.name
        assert torch.equal(fin, f_ref), w.name
        if stride:
            assert torch.equal(snaps, s_ref), w.name


def test_static_scratch_rejects_oversized_requests():
    lib = gdn.load_library()
    d = gdn.make_desc(4, 40000, 16, 128, 128, gdn.GDN_BF16, False, 1.0)
    fake = [ctypes.c_void_p(1 << 40) for _ in range(7)]
    st = lib.gdn_chunk_fwd_static(ctypes.byref(d), *fake[:5], None, None, 4, 0, fake[5], fake[6], None, None)
    assert st == gdn.GDN_ERR_WORKSPACE
    assert "scratch" in lib.gdn_last_error().decode()


_FRESH = r'''
import sys, torch
sys.path.insert(0, sys.argv[1])
from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import Workload, make_inputs
from tests.gpu_util import to_dev
w = Workload("no-alloc fresh", B=1, T=8192, H=2, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=45)
dx = to_dev(make_inputs(w))
out = torch.empty_like(dx.v)
fin = torch.empty_like(dx.h0)
# the kernels' first launches (module loading) happen in a workspace call first
ws = torch.empty(gdn.gdn_chunk_workspace_size(1, 8192, 2, 128, 128, 1), dtype=torch.uint8, device="cuda")
need = ws.numel()
gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0, out=out, final_state=fin, workspace=ws)
torch.cuda.synchronize()
del ws
torch.cuda.empty_cache()
gdn.gdn_chunk_status_static()   # the library looks up the array's address (its module loads)
torch.cuda.synchronize()
free0 = torch.cuda.mem_get_info()[0]
gdn.gdn_chunk_fwd_static(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0, out=out, final_state=fin)
torch.cuda.synchronize()
free1 = torch.cuda.mem_get_info()[0]
print(need, free0 - free1)
'''


def test_first_static_call_allocates_no_device_memory():
    r = subprocess.run([sys.executable, "-c", _FRESH, ROOT], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    need, used = (int(v) for v in r.stdout.split()[-2:])
    assert need > 16 << 20            # an allocation of the scratch would show
    assert abs(used) < 2 << 20, used  # nothing was allocated by the call
