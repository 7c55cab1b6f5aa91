"""The bounds-checked build (libgdn_checked.so, -DGDN_CHECKED) on the small parity
cases: every chunked path -- tensor cores with one gate per head and per channel,
packed sequences, the split scan with snapshots, the fp32 CUDA-core path with
d = 64 and mixed head sizes -- runs its range checks, matches the oracle, and
leaves the status word at GDN_DEV_OK.  Run in a child process that loads the
checked library through GDN_LIBRARY (the parent keeps the ordinary one)."""
import os
import subprocess
import sys

import pytest

from gated_delta_rule_64_b200 import build as gdn_build

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r'''
import sys, torch
sys.path.insert(0, sys.argv[1])
from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import Workload, make_inputs
from tests.gpu_util import check_against_oracle, rel_l2, run_oracle, tolerances, to_dev
assert gdn.LIB_PATH.endswith("libgdn_checked.so")
S = Workload("checked", B=2, T=300, H=3, dk=128, dv=128, dtype="bf16", h0_std=0.1, seed=80)
cases = [(S, None, 0), (S.replace(per_channel=True, seed=81), None, 0),
         (S.replace(seed=82), [70, 1, 300, 0, 129], 0),
         (S.replace(B=1, T=8192, H=2, seed=83), None, 1024),
         (S.replace(dtype="f32", dk=64, dv=64, seed=84), None, 0),
         (S.replace(dtype="f32", dk=128, dv=64, per_channel=True, seed=85), None, 128)]
for w, lengths, stride in cases:
    x = make_inputs(w, lengths=lengths)
    dx = to_dev(x)
    ws = torch.empty(gdn.gdn_chunk_workspace_size(*dx.q.shape[:3], w.dk, w.dv, x.n_seqs, dtype=dx.q.dtype,
                                                  per_channel=w.per_channel), dtype=torch.uint8, device="cuda")
    out, fin, snaps = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0, dx.cu_seqlens, snapshot_stride=stride,
                                        workspace=ws)
    assert gdn.gdn_chunk_status(ws) == (gdn.GDN_OK, gdn.GDN_DEV_OK), w
    check_against_oracle(x, out, fin)
    if stride:
        _, _, s_ref = run_oracle(x, snapshot_stride=stride)
        assert rel_l2(snaps, s_ref) <= tolerances(dx.q.dtype)[1]
print("checked ok", len(cases))
'''


def test_checked_build_on_the_small_cases():
    lib = gdn_build.build(checked=True)
    env = dict(os.environ, GDN_LIBRARY=lib)
    r = subprocess.run([sys.executable, "-c", _CHILD, ROOT], capture_output=True, text=True, timeout=900, cwd=ROOT,
                       env=env)
    assert r.returncode == 0, r.stderr[-3000:]
    assert "checked ok 6" in r.stdout
