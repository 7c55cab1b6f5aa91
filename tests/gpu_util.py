"""Helpers for the GPU parity tests: run the library and the oracle on the same
seeded inputs and compare."""
import os

import numpy as np
import torch

import oracle
from gated_delta_rule_64_b200 import gdn
from gated_delta_rule_64_b200.inputs import Inputs

# Tolerances: relative L2 error over the whole tensor, accumulated in fp64.
TOL_F32 = 1e-4          # fp32 inputs: outputs and states
TOL_BF16_OUT = 2e-2     # bf16 inputs: outputs
TOL_BF16_STATE = 1e-2   # bf16 inputs: final states and snapshots


def rel_l2(x, ref) -> float:
    x = np.asarray(x.detach().to("cpu", torch.float64).numpy() if isinstance(x, torch.Tensor) else x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    assert np.all(np.isfinite(x)), "non-finite values in the GPU result"
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 1e-30 else float(num)


def tolerances(dtype):
    return (TOL_F32, TOL_F32) if dtype == torch.float32 else (TOL_BF16_OUT, TOL_BF16_STATE)


def to_dev(x: Inputs, device="cuda"):
    d = lambda t: None if t is None else t.to(device).contiguous()
    return Inputs(q=d(x.q), k=d(x.k), v=d(x.v), g=d(x.g), beta=d(x.beta), h0=d(x.h0),
                  cu_seqlens=d(x.cu_seqlens), workload=x.workload)


def run_gpu(x: Inputs, *, scale=1.0, snapshot_stride=0):
    dx = to_dev(x)
    out, fin, snaps = gdn.gdn_chunk_fwd(dx.q, dx.k, dx.v, dx.g, dx.beta, dx.h0, dx.cu_seqlens, scale=scale,
                                        snapshot_stride=snapshot_stride)
    torch.cuda.synchronize()
    return out, fin, snaps


def run_oracle(x: Inputs, *, scale=1.0, snapshot_stride=0, heads=None):
    sel = (lambda t: t) if heads is None else (lambda t: t[:, :, heads])
    h0 = None if x.h0 is None else (x.h0 if heads is None else x.h0[:, heads])
    return oracle.gated_delta_rule(sel(x.q), sel(x.k), sel(x.v), sel(x.g), sel(x.beta), h0, x.cu_seqlens,
                                   scale=scale, snapshot_stride=snapshot_stride)


def check(x: Inputs, *, scale=1.0, snapshot_stride=0, heads=None):
    out, fin, snaps = run_gpu(x, scale=scale, snapshot_stride=snapshot_stride)
    o_ref, f_ref, s_ref = run_oracle(x, scale=scale, snapshot_stride=snapshot_stride, heads=heads)
    if heads is not None:
        out, fin = out[:, :, heads], fin[:, heads]
        snaps = None if snaps is None else snaps[:, :, heads]
    tol_o, tol_s = tolerances(x.q.dtype)
    eo, ef = rel_l2(out, o_ref), rel_l2(fin, f_ref)
    es = rel_l2(snaps, s_ref) if snapshot_stride else 0.0
    report = os.environ.get("GDN_PARITY_REPORT")
    if report:  # optional record of the measured errors, one line per check
        with open(report, "a") as f:
            f.write(f"{os.environ.get('PYTEST_CURRENT_TEST', '?').split(' ')[0]}\t{eo:.3e}\t{ef:.3e}\t{es:.3e}\n")
    assert eo <= tol_o and ef <= tol_s and es <= tol_s, f"rel-L2 out {eo:.2e} state {ef:.2e} snaps {es:.2e}"
    return eo, ef, es


def check_against_oracle(x: Inputs, out, fin, *, scale=1.0):
    """Outputs and final states of a GPU call on `x` against the oracle."""
    torch.cuda.synchronize()
    o_ref, f_ref, _ = run_oracle(x, scale=scale)
    tol_o, tol_s = tolerances(x.q.dtype)
    eo, ef = rel_l2(out, o_ref), rel_l2(fin, f_ref)
    assert eo <= tol_o and ef <= tol_s, f"rel-L2 out {eo:.2e} state {ef:.2e}"
    return eo, ef
