"""Host logic of bench.py (CPU): the recorded ncu traffic of a kernel is reported
only while the kernel's source text and the files it depends on are unchanged; the
SM clock record covers the timed region only."""
import hashlib
import importlib.util
import json
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


KERNEL = """// a comment
template <int N>
__global__ void __launch_bounds__(128) my_kernel(float *x) {
    x[threadIdx.x] = N;
}

__global__ void other(float *x) { x[0] = 1.f; }
"""


def _tree(tmp_path, kernel_src, dep_text):
    (tmp_path / "profiles").mkdir(exist_ok=True)
    (tmp_path / "k.cu").write_text(kernel_src)
    (tmp_path / "dep.cuh").write_text(dep_text)
    return tmp_path


def test_traffic_follows_the_kernel_source(bench, tmp_path, monkeypatch):
    root = _tree(tmp_path, KERNEL, "// helpers v1\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_hash(str(root / "k.cu"), "my_kernel")
    assert sha is not None
    rec = {"wl": {"my_kernel": {"source": "k.cu", "sha256": sha, "bytes_per_launch": 1234.0,
                                "deps": {"dep.cuh": hashlib.sha256(b"// helpers v1\n").hexdigest()}}}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(rec))
    assert bench.traffic_for("my_kernel", "wl") == 1234.0
    assert bench.traffic_for("my_kernel", "other workload") is None
    assert bench.traffic_for("missing_kernel", "wl") is None

    # text outside the kernel (a comment, another kernel) does not matter
    (root / "k.cu").write_text(KERNEL.replace("// a comment", "// another comment").replace("1.f", "2.f"))
    assert bench.traffic_for("my_kernel", "wl") == 1234.0
    # the kernel's own text does, launch bounds included
    (root / "k.cu").write_text(KERNEL.replace("x[threadIdx.x] = N;", "x[threadIdx.x] = 2 * N;"))
    assert bench.traffic_for("my_kernel", "wl") is None
    (root / "k.cu").write_text(KERNEL.replace("__launch_bounds__(128)", "__launch_bounds__(256)"))
    assert bench.traffic_for("my_kernel", "wl") is None
    # and so does every file the kernel's code comes from
    (root / "k.cu").write_text(KERNEL)
    assert bench.traffic_for("my_kernel", "wl") == 1234.0
    (root / "dep.cuh").write_text("// helpers v2\n")
    assert bench.traffic_for("my_kernel", "wl") is None


def test_committed_records_name_existing_kernels(bench):
    from gated_delta_rule_64_b200.inputs import WORKLOADS
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        records = json.load(f)
    for workload, kernels in records.items():
        assert workload in WORKLOADS, workload
        for name, rec in kernels.items():
            assert os.path.exists(os.path.join(ROOT, rec["source"])), name
            fn = rec.get("function", name)
            assert bench.kernel_source_hash(os.path.join(ROOT, rec["source"]), fn) is not None, name
            # current while the kernel's sources are unchanged, else not reported
            assert bench.traffic_for(name, workload) in (rec["bytes_per_launch"], None), (workload, name)
            assert rec["bytes_per_launch"] > 0 and rec["ncu"].startswith("ncu "), name
            assert "--clock-control none" in rec["ncu"], name
            for dep in rec.get("deps", {}):
                assert os.path.exists(os.path.join(ROOT, dep)), (name, dep)


def test_algorithmic_work_of_the_headline_workload(bench):
    """Bytes and flops the roofline divides by, for the long single-sequence workload:
    q, k, v in and o out in bf16, fp32 gate and beta per head-token, no initial state,
    the final state and 32 snapshots of 16 x 128 x 128 fp32."""
    import torch

    from gated_delta_rule_64_b200.inputs import Inputs, LONG_SNAPSHOTS
    T, H = 1024, 16  # shapes only (a shortened sequence)
    z = lambda *s, dt=torch.bfloat16: torch.empty(s, dtype=dt)
    x = Inputs(q=z(1, T, H, 128), k=z(1, T, H, 128), v=z(1, T, H, 128), g=z(1, T, H, dt=torch.float32),
               beta=z(1, T, H, dt=torch.float32), h0=None)
    w = LONG_SNAPSHOTS.replace(T=T, snapshot_stride=256)
    nbytes, flops = bench.alg_work(x, w)
    state = 128 * 128 * 4
    assert nbytes == T * H * (4 * 128 * 2 + 8) + (1 + T // 256) * H * state
    assert flops == T * H * (10 * 64 * 128 + 6 * 128 * 128 + 2 * 64 * 64 / 3)


def test_clock_samples_keep_milliseconds_and_stay_inside_the_timed_region(bench):
    text = "\n".join([
        "2026/12/02 22:20:00.100, 0, 1965, 1965, 250.0, Not Active, Not Active, Not Active, Not Active, Not Active",
        "2026/12/02 22:20:00.500, 0, 1800, 1965, 700.0, Active, Not Active, Not Active, Not Active, Active",
        "2026/12/02 22:20:00.600, 0, 1700, 1965, [N/A], Active, Not Active, Not Active, Not Active, Active",
        "2026/12/02 22:20:00.900, 0, 1965, 1965, 260.0, Not Active, Not Active, Not Active, Not Active, Not Active",
    ])
    rows = bench.parse_smi_rows(text)
    assert len(rows) == 4 and abs((rows[1][0] - rows[0][0]) - 0.4) < 1e-6
    t0 = rows[0][0] + 0.3
    out = bench.ClockSampler.summarize(rows, t0, t0 + 0.4)
    assert out["samples"] == 2 and out["sm_mhz"] == 1750 and out["sm_min_mhz"] == 1700
    assert out["reasons"] == ["sw_power_cap"] and out["power_w_max"] == 700.0
