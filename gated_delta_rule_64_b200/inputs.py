"""Seeded synthetic inputs for the gated delta rule.

This module is shared by the CUDA path's tests/benchmark and by the oracle's
tests.  It holds no arithmetic of the method itself: it only draws random
numbers and shapes them the way the layer's inputs arrive.

Recipe (all draws from ``numpy.random.default_rng(seed)``, in this order):
  1. lengths of packed sequences, when the workload is a packed batch
     (integers drawn uniformly from the workload's closed range);
  2. q, k ~ N(0, 1) per element, then each token's d_k vector is divided by its
     L2 norm in fp32 (the layer L2-normalises queries and keys: "Attention,
     Part 4", section 6, "Where alpha and beta come from");
  3. v ~ N(0, 1);
  4. beta = sigmoid(x), x ~ N(beta_mu, 1)   (computed in fp64, stored fp32);
  5. g = log(alpha) = -softplus(x), x ~ N(gate_mu, 1), one value per head and
     token, or one per key channel for the per-channel (KDA) variant;
     computed in fp64 and stored fp32 -- the library takes the gate as a log;
  6. the initial state ~ N(0, h0_std^2) when the workload has one.
q, k, v are then rounded to the workload's dtype (round-to-nearest-even for
bf16); gates, beta and states stay fp32.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int = 1
    T: int = 256
    H: int = 2
    dk: int = 64
    dv: int = 64
    dtype: str = "f32"            # "f32" or "bf16" for q, k, v and the output
    per_channel: bool = False     # KDA per-key-channel gate
    h0_std: float = 0.0           # 0: zero initial state
    snapshot_stride: int = 0
    packed_lengths: tuple | None = None   # (n_seqs, lo, hi): lengths ~ U{lo..hi}, packed
    decode_steps: int = 0         # >0: a decode workload of this many single-token steps
    gate_mu: float = -2.0
    beta_mu: float = 0.0
    chunk: int = 64
    seed: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "f32" else torch.bfloat16


# The five workloads of the benchmark suite, with the sizes and value
# distributions given for this path.  Seeds: the first is 0, the others count on.
TINY_F32 = Workload("tiny-f32 B1 H2 T256 d64", B=1, T=256, H=2, dk=64, dv=64, dtype="f32", seed=0)
PREFILL_BF16 = Workload("prefill B4 T4096 H16 d128 bf16", B=4, T=4096, H=16, dk=128, dv=128,
                        dtype="bf16", h0_std=0.02, seed=1)
LONG_SNAPSHOTS = Workload("long T262144 H16 d128 bf16 snapshots/8192", B=1, T=262144, H=16, dk=128,
                          dv=128, dtype="bf16", snapshot_stride=8192, seed=2)
KDA_PACKED = Workload("kda packed 8x[512,16384] H32 d128 bf16", B=1, T=0, H=32, dk=128, dv=128,
                      dtype="bf16", per_channel=True, h0_std=0.02, packed_lengths=(8, 512, 16384),
                      seed=3)
DECODE = Workload("decode 256 seqs x H32 d128, 64 steps", B=256, T=1, H=32, dk=128, dv=128,
                  dtype="bf16", h0_std=0.02, decode_steps=64, seed=4)

WORKLOADS = {w.name: w for w in (TINY_F32, PREFILL_BF16, LONG_SNAPSHOTS, KDA_PACKED, DECODE)}


def _sigmoid64(x):
    return 1.0 / (1.0 + np.exp(-x))


def _neg_softplus64(x):
    return -np.logaddexp(0.0, x)


def _normal(rng, shape):
    return rng.standard_normal(size=shape, dtype=np.float32)


def _unit_rows(a: np.ndarray) -> np.ndarray:
    n = np.sqrt(np.sum(a * a, axis=-1, keepdims=True, dtype=np.float32), dtype=np.float32)
    return a / np.maximum(n, np.float32(1e-30))


def draw_lengths(w: Workload) -> np.ndarray:
    n, lo, hi = w.packed_lengths
    rng = np.random.default_rng(w.seed)
    return rng.integers(lo, hi + 1, size=n, dtype=np.int64)


@dataclass
class Inputs:
    """CPU tensors in the library's layout.

    q, k: (B, T, H, dk); v: (B, T, H, dv) -- workload dtype
    g:    (B, T, H) or (B, T, H, dk) fp32, the log of the decay gate
    beta: (B, T, H) fp32
    h0:   (N, H, dv, dk) fp32 or None
    cu_seqlens: (N+1,) int32 offsets into the B*T rows, or None
    For decode workloads every tensor but h0 has a leading step axis and T = 1.
    """
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    h0: torch.Tensor | None
    cu_seqlens: torch.Tensor | None = None
    workload: Workload | None = None
    extra: dict = field(default_factory=dict)

    @property
    def n_seqs(self) -> int:
        return (self.cu_seqlens.numel() - 1) if self.cu_seqlens is not None else self.q.shape[-4]

    def tokens(self) -> int:
        return int(self.q.shape[-4] * self.q.shape[-3]) if self.cu_seqlens is None else int(self.cu_seqlens[-1])


def make_inputs(w: Workload, *, lengths=None, heads: int | None = None) -> Inputs:
    """Draw the inputs of workload `w` (see the module docstring for the recipe).

    `lengths` overrides the packed lengths; `heads` overrides H (for reduced
    test sizes with the same distributions).
    """
    rng = np.random.default_rng(w.seed)
    H = heads or w.H
    cu = None
    if w.packed_lengths is not None or lengths is not None:
        if lengths is None:
            n, lo, hi = w.packed_lengths
            lengths = rng.integers(lo, hi + 1, size=n, dtype=np.int64)  # same draw as draw_lengths
        lengths = np.asarray(lengths, dtype=np.int64)
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        B, T = 1, int(cu[-1])
    else:
        B, T = w.B, w.T
    lead = (w.decode_steps,) if w.decode_steps else ()
    N = len(cu) - 1 if cu is not None else B

    q = _unit_rows(_normal(rng, lead + (B, T, H, w.dk)))
    k = _unit_rows(_normal(rng, lead + (B, T, H, w.dk)))
    v = _normal(rng, lead + (B, T, H, w.dv))
    beta = _sigmoid64(rng.standard_normal(size=lead + (B, T, H)) + w.beta_mu).astype(np.float32)
    gshape = lead + ((B, T, H, w.dk) if w.per_channel else (B, T, H))
    g = _neg_softplus64(rng.standard_normal(size=gshape) + w.gate_mu).astype(np.float32)
    h0 = None
    if w.h0_std > 0:
        h0 = (_normal(rng, (N, H, w.dv, w.dk)) * np.float32(w.h0_std)).astype(np.float32)

    td = w.torch_dtype
    return Inputs(
        q=torch.from_numpy(q).to(td), k=torch.from_numpy(k).to(td), v=torch.from_numpy(v).to(td),
        g=torch.from_numpy(g), beta=torch.from_numpy(beta),
        h0=None if h0 is None else torch.from_numpy(h0),
        cu_seqlens=None if cu is None else torch.from_numpy(cu),
        workload=w.replace(H=H))


@dataclass
class PreruleInputs:
    """Raw projections of a Gated DeltaNet layer (CPU tensors): x (B, T, C) with
    C = 2 hk dk + H dv, a and b (B, T, H) in `dtype`; conv_w (C, K), A_log and
    dt_bias (H,) and an optional convolution history (N, C, K-1) in fp32."""
    x: torch.Tensor
    a: torch.Tensor
    b: torch.Tensor
    conv_w: torch.Tensor
    A_log: torch.Tensor
    dt_bias: torch.Tensor
    hist: torch.Tensor | None
    cu_seqlens: torch.Tensor | None
    hk: int
    dk: int
    H: int
    dv: int


def make_prerule_inputs(*, B, T, H, hk, dk, dv, K=4, dtype="bf16", lengths=None, history=True,
                        seed=0) -> PreruleInputs:
    """Seeded raw projections, drawn in this order: packed lengths (if any), x ~ N(0,1),
    a ~ N(0,1), b ~ N(0,1), conv_w ~ N(0, 1/K), A_log ~ U(0, log 16), dt_bias ~ N(0, 0.25),
    history ~ N(0,1).  Values are rounded to `dtype` where the layer holds them in it."""
    rng = np.random.default_rng(seed)
    cu = None
    if lengths is not None:
        lengths = np.asarray(lengths, dtype=np.int64)
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
        B, T = 1, int(cu[-1])
    N = len(cu) - 1 if cu is not None else B
    C = 2 * hk * dk + H * dv
    x = _normal(rng, (B, T, C))
    a = _normal(rng, (B, T, H))
    b = _normal(rng, (B, T, H))
    conv_w = (_normal(rng, (C, K)) / np.float32(np.sqrt(K))).astype(np.float32)
    A_log = rng.uniform(0.0, np.log(16.0), size=H).astype(np.float32)
    dt_bias = (rng.standard_normal(H) * 0.5).astype(np.float32)
    hist = _normal(rng, (N, C, K - 1)) if history else None
    td = torch.float32 if dtype == "f32" else torch.bfloat16
    t = lambda z: torch.from_numpy(z)
    return PreruleInputs(x=t(x).to(td), a=t(a).to(td), b=t(b).to(td), conv_w=t(conv_w), A_log=t(A_log),
                         dt_bias=t(dt_bias), hist=None if hist is None else t(hist),
                         cu_seqlens=None if cu is None else t(cu), hk=hk, dk=dk, H=H, dv=dv)
