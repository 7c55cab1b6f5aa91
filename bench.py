"""Throughput of the gated delta rule on B200: chunked prefill (headline) and decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one chunked-prefill pass (gdn_chunk_fwd) over the long single-sequence
workload: one sequence of T=262,144 tokens, H=16 heads, d_k=d_v=128 (bf16 q/k/v,
fp32 gates and states, chunk 64), zero initial state, a state snapshot every 8,192
tokens (32 of them) and the final state.  `value` is prefill tokens/s over all
ranks (every rank runs its own sequence: weak scaling, no collective on the data
path), timed with CUDA events around exactly K steps after W warm-up steps, max
over ranks.  The inputs (~3.2 GB) are larger than L2, so no explicit flush is
done between steps.

The same line carries:
  e2e          the same metric with host (pinned) inputs copied in and the
               outputs (o, final state, snapshots) copied back inside the timed
               region (consecutive steps pipelined over three streams);
  roofline     HBM roofline of the step (algorithmic bytes over the summed
               device time of its kernels, from the library's own per-kernel
               event timer in the timed region), its tensor-core counterpart,
               and per kernel its time, share and recorded DRAM traffic;
  prefill_b4   the same for the prefill workload B=4, T=4096, H=16;
  kda_packed   the same for the per-channel-gate workload (8 packed sequences
               of 512..16384 tokens, H=32);
  decode       decode tokens/s on 256 sequences x 32 heads (state updated in
               place, 64 steps per pass) with its own roofline;
  cpu_baseline the fp64 oracle on a bounded sample of the headline workload,
               on this host's cores (one thread per head);
  clocks       SM clocks sampled with nvidia-smi during the headline's timed region.

--impl reference times the oracle (the CPU reference of the method) instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "gated-delta-rule prefill tokens/s & decode tokens/s, % of TC/HBM roofline"
UNIT = "tokens/s"

# Algorithmic traffic and work of the prefill workload, per head-token.
# bytes: q, k, v in and o out (bf16, 128 each) + fp32 gate and beta;
# states (initial read + final write, 2 x 64 KiB per (sequence, head)) are added per unit.
PREFILL_BYTES_PER_HEAD_TOKEN = 4 * 128 * 2 + 4 + 4
STATE_BYTES = 128 * 128 * 4
# flops: 10*C*d + 6*d^2 + 2*C^2/3 per head-token for C = 64, d = 128
PREFILL_FLOPS_PER_HEAD_TOKEN = 10 * 64 * 128 + 6 * 128 * 128 + 2 * 64 * 64 / 3
# decode, per (sequence, head) and step: fp32 state read + written, q/k/v/o bf16, gate+beta fp32
DECODE_BYTES_PER_UNIT = 2 * STATE_BYTES + 4 * 128 * 2 + 4 + 4


def env_rank():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------------------
# Clock sampling
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return self.summarize(parse_smi_rows(out), self.t0, self.t1)

    @staticmethod
    def summarize(rows, t0, t1):
        """Median SM clock (and the lowest) over the samples taken inside [t0, t1]."""
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        inside = [r for r in rows if t0 is not None and t0 <= r[0] <= (t1 if t1 is not None else r[0])]
        if not inside and t0 is not None:  # a region shorter than the sampling period
            inside = [r for r in rows if t0 - 0.2 <= r[0] <= (t1 if t1 is not None else t0) + 0.2]
        use = inside or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[3][1:]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_min_mhz": min(r[1] for r in use),
                "sm_max_mhz": max(r[2] for r in use),
                "power_w_max": max((r[4] for r in use if r[4] == r[4]), default=None),
                "reasons": reasons, "samples": len(use)}


def parse_smi_rows(text):
    """(time, clocks.sm, clocks.max.sm, reason flags, power.draw) per line of the sampler's output;
    the timestamp keeps its milliseconds."""
    rows = []
    for line in text.strip().splitlines():
        parts = [p.strip() for p in line.split(",")]
        if len(parts) < 10:
            continue
        try:
            whole, _, frac = parts[0].partition(".")
            ts = time.mktime(time.strptime(whole, "%Y/%m/%d %H:%M:%S")) + (float("0." + frac) if frac.isdigit() else 0.0)
            try:
                power = float(parts[4])
            except ValueError:  # "[N/A]"
                power = float("nan")
            rows.append((ts, float(parts[2]), float(parts[3]), parts[5:10], power))
        except ValueError:
            continue
    return rows


# ---------------------------------------------------------------------------
# Multi-rank plumbing (host logic; tested with gloo on CPU)
# ---------------------------------------------------------------------------
def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own batch of the workload (independent sequences)."""
    return base + 1000 * rank


# ---------------------------------------------------------------------------
# Oracle (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(tokens_per_seq: int):
    """The first `tokens_per_seq` tokens of the long single-sequence workload (all 16
    heads; its zero initial state), drawn as the full workload would be."""
    from gated_delta_rule_64_b200.inputs import LONG_SNAPSHOTS, make_inputs
    w = LONG_SNAPSHOTS.replace(T=tokens_per_seq, snapshot_stride=0)
    return w, make_inputs(w)


def time_oracle(x, n_threads):
    import oracle
    t = time.perf_counter()
    oracle.gated_delta_rule(x.q, x.k, x.v, x.g, x.beta, x.h0, n_threads=n_threads)
    return time.perf_counter() - t


def oracle_threads() -> int:
    """Threads the oracle uses on this host: one per (sequence, head) unit at most."""
    import oracle
    return max(1, min(oracle.host_threads(), 16))


def sample_tokens(budget_s: float, cores: int) -> int:
    """Tokens of the long sequence the oracle gets through in about `budget_s` seconds."""
    _, x = oracle_sample(256)
    per_tok = time_oracle(x, cores) / 256
    return int(max(256, min(262144, budget_s / per_tok)) // 64 * 64)


def cpu_baseline(target_s: float = 12.0):
    cores = oracle_threads()
    T = sample_tokens(target_s, cores)
    _, x = oracle_sample(T)
    dt = time_oracle(x, cores)
    return {"value": T / dt, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
            "sample": f"long single-sequence workload (T=262144, H=16, d=128, bf16 inputs): its first {T} tokens, "
                      f"all 16 heads, fp64 token loop, one thread per head, {dt:.1f} s"}


def run_reference(args):
    rank, world, _ = env_rank()
    if rank != 0:
        return 0
    from gated_delta_rule_64_b200.inputs import LONG_SNAPSHOTS
    cores = oracle_threads()
    budget = 150.0
    T = sample_tokens(budget / max(1, args.steps + args.warmup), cores)
    _, x = oracle_sample(T)
    for _ in range(args.warmup):
        time_oracle(x, cores)
    times = [time_oracle(x, cores) for _ in range(args.steps)]
    dt = sum(times) / len(times)
    value = T / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": LONG_SNAPSHOTS.name + " (bounded sample per step)", "global_batch": 1,
                   "seq_len": LONG_SNAPSHOTS.T, "parallelism": "replicas only: oracle on rank 0",
                   "sample_tokens": T},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "cpu_model": cpu_model(), "kind": "oracle",
                         "sample": f"first {T} tokens of the sequence, all 16 heads, per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def kernel_source_hash(path: str, name: str):
    """sha256 of the source text of the __global__ function `name` in `path`."""
    if not os.path.exists(path):
        return None
    text = open(path).read()
    i = text.find(f"\n{name}(")
    if i < 0:
        i = text.find(f" {name}(")
    if i < 0:
        return None
    start = text.rfind("__global__", 0, i)
    end = text.find("\n}\n", i)
    if start < 0 or end < 0:
        return None
    return hashlib.sha256(text[start:end].encode()).hexdigest()


def traffic_for(kernel: str, workload: str):
    """ncu DRAM bytes (read + write) per launch of `kernel` on `workload`, as recorded in
    profiles/traffic.json ({workload: {kernel: record}}), or None when there is no
    record or the kernel's source (or a file it depends on) changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p)).get(workload, {}).get(kernel)
    if not rec:
        return None
    # (`kernel` is the library's timer label; the record names the __global__ function)
    if kernel_source_hash(os.path.join(ROOT, rec["source"]), rec.get("function", kernel)) != rec["sha256"]:
        return None
    for dep, sha in rec.get("deps", {}).items():  # files the kernel's code comes from, hashed whole
        path = os.path.join(ROOT, dep)
        if not os.path.exists(path) or hashlib.sha256(open(path, "rb").read()).hexdigest() != sha:
            return None
    return float(rec["bytes_per_launch"])


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def alg_work(x, w):
    """Algorithmic bytes and flops of one chunked-prefill pass over inputs `x` of workload `w`:
    q, k, v read and o written once (their dtype), the fp32 gate (per head or per key
    channel) and beta read once, the initial state read (when given), the final state
    and the snapshots written once; flops per head-token as in the chunkwise form."""
    el = x.q.element_size()
    H, dk, dv = x.v.shape[2], x.q.shape[3], x.v.shape[3]
    N = x.n_seqs
    n_snap = (x.q.shape[1] // w.snapshot_stride) if w.snapshot_stride else 0
    head_tokens = x.tokens() * H
    per_ht = (2 * dk + 2 * dv) * el + 4 * (dk if w.per_channel else 1) + 4
    states = ((1 if x.h0 is not None else 0) + 1 + n_snap) * N * H * dv * dk * 4
    return head_tokens * per_ht + states, head_tokens * PREFILL_FLOPS_PER_HEAD_TOKEN


def time_chunked(w, args, rank, world, dev, pk, *, clocks=None, e2e=False):
    """Time K chunked-prefill steps of workload `w` (every rank its own seeded batch),
    with the library's per-kernel event timer on; optionally the end-to-end metric
    through host buffers.  Returns (result dict, device tensors kept for nothing)."""
    import torch
    import torch.distributed as dist

    from gated_delta_rule_64_b200 import gdn
    from gated_delta_rule_64_b200.inputs import make_inputs

    w = w.replace(seed=rank_seed(w.seed, rank))
    x = make_inputs(w)
    d = lambda t: None if t is None else t.to(dev).contiguous()
    q, k, v, g, beta, h0, cu = d(x.q), d(x.k), d(x.v), d(x.g), d(x.beta), d(x.h0), d(x.cu_seqlens)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    N = x.n_seqs
    n_snap = T // w.snapshot_stride if w.snapshot_stride else 0
    out = torch.empty((B, T, H, dv), dtype=q.dtype, device=dev)
    fin = torch.empty((N, H, dv, dk), dtype=torch.float32, device=dev)
    snaps = torch.empty((N, n_snap, H, dv, dk), dtype=torch.float32, device=dev) if n_snap else None
    ws = torch.empty(gdn.gdn_chunk_workspace_size(B, T, H, dk, dv, N, dtype=q.dtype, per_channel=w.per_channel),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(bufs=None, s=stream):
        bq, bk, bv, bg, bb, bh0, bout, bfin, bsn, bws = bufs or (q, k, v, g, beta, h0, out, fin, snaps, ws)
        gdn.gdn_chunk_fwd(bq, bk, bv, bg, bb, bh0, cu, snapshot_stride=w.snapshot_stride, out=bout,
                          final_state=bfin, snapshots=bsn, workspace=bws, stream=s)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, code = gdn.gdn_chunk_status(ws)
    if st != gdn.GDN_OK:
        raise RuntimeError(f"{w.name}: device status {code}")
    gdn.profile_read()
    gdn.profile_enable(True)
    barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark_begin()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    if clocks:
        clocks.mark_end()
    barrier()
    gdn.profile_enable(False)
    kernels = gdn.profile_read()
    ms_step = max_over_ranks(e0.elapsed_time(e1), world, dev) / args.steps
    tokens = x.tokens()
    value = tokens * world / (ms_step * 1e-3)

    # Roofline of the step.  The chunked prefill is two to four kernels (chunk-local
    # work on every chunk in parallel, then the ordered scan in one or two passes);
    # none of them moves the path's algorithmic bytes on its own, so the HBM roofline
    # is taken over the step: algorithmic bytes / summed kernel time.
    alg_bytes, alg_flops = alg_work(x, w)
    per_step = {n: t / args.steps * 1e-3 for n, (c, t) in kernels.items()}  # seconds per step, per kernel
    launches = {n: c / args.steps for n, (c, t) in kernels.items()}
    step_s = sum(per_step.values()) or ms_step * 1e-3
    achieved = alg_bytes / step_s / 1e9
    traffics = {n: traffic_for(n, w.name) for n in per_step}
    traffic = (sum(traffics[n] * launches[n] for n in per_step)
               if traffics and all(t is not None for t in traffics.values()) else None)
    top = max(per_step, key=per_step.get) if per_step else "none"
    roofline = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / pk["hbm_gbs"], "traffic": traffic,
                "scope": "one prefill step: algorithmic bytes / summed kernel time (" + " + ".join(sorted(per_step))
                         + ")",
                "algorithmic_bytes": alg_bytes, "peak_source": f"{pk['source']} hbm_gbs (burst copy)",
                "tensor": {"algorithmic_flops": alg_flops, "achieved_tflops": alg_flops / step_s / 1e12,
                           "peak": pk["bf16_tflops"], "frac": alg_flops / step_s / 1e12 / pk["bf16_tflops"],
                           "peak_source": f"{pk['source']} bf16_tflops (burst)"},
                "kernels": {n: {"launches_per_step": launches[n], "us_per_step": per_step[n] * 1e6,
                                "share": per_step[n] / step_s, "traffic_per_launch": traffics[n]}
                            for n in per_step},
                "dominant_kernel": top}
    res = {"value": value, "unit": UNIT, "ms_per_step": ms_step, "tokens_per_step": tokens * world,
           "config": {"workload": w.name, "sequences": N, "tokens": tokens, "heads": H, "d_k": dk, "d_v": dv,
                      "per_channel_gate": w.per_channel, "snapshot_stride": w.snapshot_stride, "chunk": 64},
           "roofline": roofline, "gpu_launches": sum(c for c, _ in kernels.values())}

    if e2e:
        # Every step copies its inputs in from pinned host memory, runs gdn_chunk_fwd and
        # copies its outputs (o, final state, snapshots) back.  Three streams and two
        # device buffer sets pipeline consecutive steps: step s+1's inputs go in while
        # step s computes and step s-1's results come out (PCIe runs both ways at once).
        pin = lambda t: None if t is None else t.pin_memory()
        hin = [pin(t) for t in (x.q, x.k, x.v, x.g, x.beta, x.h0)]
        hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (out, fin, snaps) if t is not None]
        h2d = sum(t.numel() * t.element_size() for t in hin if t is not None)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        sets = [(q, k, v, g, beta, h0, out, fin, snaps, ws)]
        sets.append(tuple(None if t is None else torch.empty_like(t) for t in sets[0]))
        s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        freed = [None, None]

        def e2e_step(i):
            b = sets[i & 1]
            if freed[i & 1] is not None:
                s_in.wait_event(freed[i & 1])
            with torch.cuda.stream(s_in):
                for src, dst in zip(hin, b[:6]):
                    if src is not None:
                        dst.copy_(src, non_blocking=True)
            landed = torch.cuda.Event()
            landed.record(s_in)
            s_comp.wait_event(landed)
            step(b, s_comp)
            done = torch.cuda.Event()
            done.record(s_comp)
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                for src, dst in zip([t for t in b[6:9] if t is not None], hout):
                    dst.copy_(src, non_blocking=True)
            freed[i & 1] = torch.cuda.Event()
            freed[i & 1].record(s_out)

        n_e2e = max(3, min(args.steps, 10))
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        e0.record(s_in)
        for i in range(n_e2e):
            e2e_step(i)
        e1.record(s_out)  # after the last step's copies back, which follow every earlier step's work
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev) / n_e2e
        res["e2e"] = {"value": tokens * world / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": n_e2e,
                      "pipelined": "3 streams, 2 buffer sets: step s+1 in, step s compute, step s-1 out"}
        del sets, hin, hout
    del q, k, v, g, beta, h0, cu, out, fin, snaps, ws
    torch.cuda.empty_cache()
    return res


def time_decode(args, rank, world, dev, pk):
    import torch

    from gated_delta_rule_64_b200 import gdn
    from gated_delta_rule_64_b200.inputs import DECODE, make_inputs

    wd = DECODE.replace(seed=rank_seed(DECODE.seed, rank))
    xd = make_inputs(wd)
    d = lambda t: t.to(dev).contiguous()
    dq, dk_, dv_, dg, db = (d(t) for t in (xd.q, xd.k, xd.v, xd.g, xd.beta))
    state = d(xd.h0)
    steps_d = xd.q.shape[0]
    dout = torch.empty((steps_d,) + tuple(xd.v.shape[1:]), dtype=dq.dtype, device=dev)
    stream = torch.cuda.current_stream()

    def decode_pass():
        for s in range(steps_d):
            gdn.gdn_decode_step(dq[s], dk_[s], dv_[s], dg[s], db[s], state, out=dout[s], stream=stream)

    decode_pass()
    torch.cuda.synchronize()
    passes = max(2, min(10, args.steps // 10 + 1))
    gdn.profile_read()
    gdn.profile_enable(True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(passes):
        decode_pass()
    e1.record(stream)
    torch.cuda.synchronize()
    gdn.profile_enable(False)
    times = gdn.profile_read()
    dms = max_over_ranks(e0.elapsed_time(e1), world, dev) / (passes * steps_d)
    nseq = xd.q.shape[1]
    units = nseq * xd.q.shape[3]
    name, (launches, total_ms) = max(times.items(), key=lambda kv: kv[1][1])
    per_launch = total_ms / launches * 1e-3
    ach = units * DECODE_BYTES_PER_UNIT / per_launch / 1e9
    del dq, dk_, dv_, dg, db, state, dout
    torch.cuda.empty_cache()
    return {"metric": "decode tokens/s", "value": nseq * world / (dms * 1e-3), "unit": UNIT, "ms_per_step": dms,
            "config": {"workload": wd.name, "sequences": nseq, "heads": xd.q.shape[3],
                       "state": "fp32 in HBM, updated in place"},
            "roofline": {"bound": "hbm", "achieved": ach, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / pk["hbm_gbs"], "traffic": traffic_for(name, wd.name), "kernel": name,
                         "algorithmic_bytes_per_launch": units * DECODE_BYTES_PER_UNIT,
                         "peak_source": f"{pk['source']} hbm_gbs (burst copy)"},
            "gpu_launches": sum(c for c, _ in times.values())}


def run_gpu(args):
    import torch
    import torch.distributed as dist

    from gated_delta_rule_64_b200 import gdn
    from gated_delta_rule_64_b200.inputs import KDA_PACKED, LONG_SNAPSHOTS, PREFILL_BF16

    rank, world, local = env_rank()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    gdn.load_library()
    pk = peaks()

    clocks = ClockSampler(local)
    clocks.start()
    head = time_chunked(LONG_SNAPSHOTS, args, rank, world, dev, pk, clocks=clocks, e2e=True)
    clk = clocks.stop()
    others = {}
    if not args.headline_only:
        others["prefill_b4"] = time_chunked(PREFILL_BF16, args, rank, world, dev, pk)
        others["kda_packed"] = time_chunked(KDA_PACKED, args, rank, world, dev, pk)
        others["decode"] = time_decode(args, rank, world, dev, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        cfg = dict(head["config"])
        cfg.update({"global_batch": cfg["sequences"] * world, "seq_len": LONG_SNAPSHOTS.T,
                    "parallelism": f"dp{world} (independent sequences per rank)" if world > 1 else "single GPU",
                    "l2": "inputs larger than L2 (no flush)"})
        line = {
            "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "roofline": head["roofline"], "cpu_baseline": cpu, "clocks": clk, "e2e": head["e2e"],
            "gpu_launches": head["gpu_launches"],
        }
        line.update(others)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


SECONDARY = {"kda": "KDA_PACKED", "long": "LONG_SNAPSHOTS", "tiny": "TINY_F32", "spec": "DECODE",
             "prerule": "PREFILL_BF16"}
SPEC_K = 4  # draft tokens per sequence in the speculative-decoding measurement


def run_prerule(args) -> int:
    """The work before the recurrence (gdn_prerule: short convolution + SiLU, q/k length,
    gates) on the prefill workload's shape, with the convolution history read and
    written, then the same followed by the chunked prefill (the layer core); and a
    decode step from raw projections on the decode workload's shape, fused
    (gdn_decode_step_prerule) and as gdn_prerule followed by gdn_decode_step."""
    import torch

    from gated_delta_rule_64_b200 import gdn
    from gated_delta_rule_64_b200.inputs import PREFILL_BF16, make_prerule_inputs

    torch.cuda.set_device(0)
    pk = peaks()
    w = PREFILL_BF16
    pi = make_prerule_inputs(B=w.B, T=w.T, H=w.H, hk=w.H, dk=w.dk, dv=w.dv, dtype=w.dtype, seed=w.seed)
    d = lambda t: t.cuda().contiguous()
    x, a, b, cw, al, dtb, hist = (d(t) for t in (pi.x, pi.a, pi.b, pi.conv_w, pi.A_log, pi.dt_bias, pi.hist))
    h0 = torch.zeros((w.B, w.H, w.dv, w.dk), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    B, T, C = x.shape
    K = cw.shape[1]
    ws = torch.empty(gdn.gdn_chunk_workspace_size(B, T, w.H, w.dk, w.dv, B), dtype=torch.uint8, device="cuda")
    res = {}
    modes = {
        "prerule": lambda: gdn.gdn_prerule(x, a, b, cw, al, dtb, hk=w.H, dk=w.dk, H=w.H, dv=w.dv,
                                           conv_state_in=hist, conv_state_out=hist, stream=stream),
        "prerule+prefill": lambda: gdn.gdn_chunk_fwd(*gdn.gdn_prerule(x, a, b, cw, al, dtb, hk=w.H, dk=w.dk, H=w.H,
                                                                      dv=w.dv, conv_state_in=hist,
                                                                      conv_state_out=hist, stream=stream),
                                                     h0, final_state=h0, workspace=ws, stream=stream),
    }
    # a decode step from raw projections on the decode workload's shape (256 sequences x
    # 32 heads, one token each): fused (gdn_decode_step_prerule) against gdn_prerule
    # followed by gdn_decode_step
    from gated_delta_rule_64_b200.inputs import DECODE
    wd = DECODE
    pd = make_prerule_inputs(B=wd.B, T=1, H=wd.H, hk=wd.H, dk=wd.dk, dv=wd.dv, dtype=wd.dtype, seed=wd.seed)
    dx, da, db, dcw, dal, ddt, dhist = (d(t) for t in (pd.x[:, 0], pd.a[:, 0], pd.b[:, 0], pd.conv_w, pd.A_log,
                                                       pd.dt_bias, pd.hist))
    dstate = torch.zeros((wd.B, wd.H, wd.dv, wd.dk), dtype=torch.float32, device="cuda")
    dout = torch.empty((wd.B, wd.H, wd.dv), dtype=dx.dtype, device="cuda")
    modes["decode: fused pre-rule + step"] = lambda: gdn.gdn_decode_step_prerule(
        dx, da, db, dcw, dal, ddt, dhist, dstate, hk=wd.H, dk=wd.dk, H=wd.H, dv=wd.dv, out=dout, stream=stream)
    modes["decode: pre-rule, then step"] = lambda: gdn.gdn_decode_step(
        *gdn.gdn_prerule(dx[:, None], da[:, None], db[:, None], dcw, dal, ddt, hk=wd.H, dk=wd.dk, H=wd.H, dv=wd.dv,
                         conv_state_in=dhist, conv_state_out=dhist, stream=stream), dstate, out=dout, stream=stream)
    tokens = {"decode: fused pre-rule + step": wd.B, "decode: pre-rule, then step": wd.B}
    el = x.element_size()
    pre_bytes = B * T * (C * el + 2 * w.H * el) + 2 * B * C * (K - 1) * 4 + B * T * C * el + B * T * w.H * 8
    clocks = ClockSampler(0)
    clocks.start()
    for name, f in modes.items():
        for _ in range(args.warmup):
            f()
        torch.cuda.synchronize()
        gdn.profile_read()
        gdn.profile_enable(True)
        clocks.mark_begin()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            f()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
        gdn.profile_enable(False)
        kern = gdn.profile_read()
        ms = e0.elapsed_time(e1) / args.steps
        res[name] = {"ms_per_step": ms, "tokens_per_s": tokens.get(name, B * T) / (ms * 1e-3),
                     "kernels_us": {n: t / max(1, c) * 1e3 for n, (c, t) in kern.items()}}
    pre_us = res["prerule"]["kernels_us"].get("gdn_prerule_kernel", 0.0) + \
        res["prerule"]["kernels_us"].get("gdn_prerule_history", 0.0)
    achieved = pre_bytes / (pre_us * 1e-6) / 1e9 if pre_us else None
    clk = clocks.stop()
    line = {"metric": "pre-rule tokens/s (secondary workload)", "value": res["prerule"]["tokens_per_s"], "unit": UNIT,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": f"raw projections of {w.name}, convolution width {K}", "channels": C},
            "modes": res,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / pk["hbm_gbs"] if achieved else None, "algorithmic_bytes": pre_bytes},
            "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def run_spec(args) -> int:
    """Speculative decoding on the decode workload's shape (256 sequences x 32 heads,
    d = 128): one gdn_decode_multi call per SPEC_K draft tokens, (a) committing all
    of them, (b) verifying without commit while writing every step's state, then
    adopting the accepted step (gdn_state_select, all drafts accepted)."""
    import torch

    from gated_delta_rule_64_b200 import gdn
    from gated_delta_rule_64_b200.inputs import DECODE, make_inputs

    torch.cuda.set_device(0)
    pk = peaks()
    w = DECODE.replace(decode_steps=0, T=SPEC_K)
    x = make_inputs(w)
    d = lambda t: t.cuda().contiguous()
    q, k, v, g, beta, h0 = d(x.q), d(x.k), d(x.v), d(x.g), d(x.beta), d(x.h0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    state = h0.clone()
    out = torch.empty_like(v)
    steps = torch.empty((B, T, H, dv, dk), dtype=torch.float32, device="cuda")
    accept = torch.full((B,), T, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    modes = {
        "commit": lambda: gdn.gdn_decode_multi(q, k, v, g, beta, state, commit=True, out=out, stream=stream),
        "verify_select": lambda: (gdn.gdn_decode_multi(q, k, v, g, beta, state, commit=False, step_states=steps,
                                                       out=out, stream=stream),
                                  gdn.gdn_state_select(steps, accept, state, stream=stream)),
    }
    tok_bytes = T * (2 * dk + 2 * dv) * q.element_size() + T * 8
    bytes_per_unit = {"commit": 2 * STATE_BYTES + tok_bytes,
                      "verify_select": STATE_BYTES + T * STATE_BYTES + tok_bytes + 2 * STATE_BYTES}
    res = {}
    clocks = ClockSampler(0)
    clocks.start()
    for name, f in modes.items():
        for _ in range(args.warmup):
            f()
        torch.cuda.synchronize()
        gdn.profile_read()
        gdn.profile_enable(True)
        clocks.mark_begin()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            f()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark_end()
        gdn.profile_enable(False)
        kern = gdn.profile_read()
        ms = e0.elapsed_time(e1) / args.steps
        achieved = B * H * bytes_per_unit[name] / (ms * 1e-3) / 1e9
        res[name] = {"ms_per_call": ms, "tokens_per_s": B * T / (ms * 1e-3), "hbm_gbs": achieved,
                     "frac": achieved / pk["hbm_gbs"], "algorithmic_bytes": B * H * bytes_per_unit[name],
                     "kernels": {n: t / max(1, c) * 1e3 for n, (c, t) in kern.items()}}
    clk = clocks.stop()
    line = {"metric": "speculative decode tokens/s (secondary workload)", "value": res["commit"]["tokens_per_s"],
            "unit": UNIT, "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": f"{w.name}: {T} tokens per sequence per call", "sequences": B, "heads": H,
                       "d_k": dk, "d_v": dv},
            "modes": res, "roofline": {"bound": "hbm", "peak": pk["hbm_gbs"], "unit": "GB/s",
                                       "achieved": res["commit"]["hbm_gbs"], "frac": res["commit"]["frac"]},
            "clocks": clk}
    print(json.dumps(line), flush=True)
    return 0


def run_secondary(args) -> int:
    """Time one of the other chunked workloads the way the headline line times its
    workload; prints one JSON line of its own (one GPU)."""
    import torch

    from gated_delta_rule_64_b200 import gdn, inputs

    w = getattr(inputs, SECONDARY[args.workload])
    torch.cuda.set_device(0)
    gdn.load_library()
    pk = peaks()
    clocks = ClockSampler(0)
    clocks.start()
    res = time_chunked(w, args, 0, 1, torch.device("cuda", 0), pk, clocks=clocks)
    res.update({"metric": "chunked prefill tokens/s (secondary workload)", "steps": args.steps,
                "warmup": args.warmup, "higher_is_better": True, "dtype": w.dtype, "data": "synthetic",
                "clocks": clocks.stop()})
    print(json.dumps(res), flush=True)
    return 0


def run_profile(which: str) -> int:
    import torch

    from gated_delta_rule_64_b200 import gdn
    from gated_delta_rule_64_b200.inputs import DECODE, KDA_PACKED, LONG_SNAPSHOTS, PREFILL_BF16, make_inputs
    d = lambda t: None if t is None else t.cuda()
    if which != "decode":
        # kda-small: the per-channel packed workload on 8 of its 32 heads (about 1.5 GB on the
        # device); long-small: the first 32768 tokens of the long sequence (about 1 GB)
        x = {"prefill": lambda: make_inputs(PREFILL_BF16), "kda-small": lambda: make_inputs(KDA_PACKED, heads=8),
             "long": lambda: make_inputs(LONG_SNAPSHOTS),
             "long-small": lambda: make_inputs(LONG_SNAPSHOTS.replace(T=32768))}[which]()
        q, k, v, g, b, h0, cu = d(x.q), d(x.k), d(x.v), d(x.g), d(x.beta), d(x.h0), d(x.cu_seqlens)
        stride = 8192 if which.startswith("long") else 0
        for _ in range(3):
            gdn.gdn_chunk_fwd(q, k, v, g, b, h0, cu, snapshot_stride=stride)
    else:
        x = make_inputs(DECODE.replace(decode_steps=3))
        st = d(x.h0)
        for s in range(3):
            gdn.gdn_decode_step(d(x.q[s]), d(x.k[s]), d(x.v[s]), d(x.g[s]), d(x.beta[s]), st)
    torch.cuda.synchronize()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="time only the headline workload (no prefill-B4 / per-channel / decode objects)")
    ap.add_argument("--profile", choices=["prefill", "decode", "kda-small", "long", "long-small"],
                    help="run three calls of one workload and exit (for ncu captures; prints nothing to time)")
    ap.add_argument("--workload", choices=["prefill"] + sorted(SECONDARY), default="prefill",
                    help="prefill (default): the headline line; kda / long / tiny: time that chunked "
                         "workload instead; spec: multi-token decode / speculative verify; prerule: the work before "
                         "the recurrence (one GPU, its own JSON line)")
    args = ap.parse_args(argv)
    if args.profile:
        return run_profile(args.profile)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.workload == "spec":
        return run_spec(args)
    if args.workload == "prerule":
        return run_prerule(args)
    if args.workload != "prefill":
        return run_secondary(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
