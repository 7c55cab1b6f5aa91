"""Host code under AddressSanitizer and UndefinedBehaviorSanitizer (CPU only).

Two executables are built here, from the committed sources, with
`-fsanitize=address,undefined -fno-sanitize-recover=all`:
  * the fp64 oracle (oracle/gdn_oracle.c) with tests/csrc/oracle_sanitize_main.c,
    which runs it over small problems through every branch (both gate kinds,
    packed sequences with an empty one, given and zero initial states,
    snapshots, the additive test mode, several threads) and over bad arguments;
  * the C-ABI library (every csrc/*.cu; the sanitizers instrument its host code:
    validation, workspace planning, the split choice, error strings, the event
    timer) with tests/csrc/abi_sanitize_main.c, which drives every entry point
    with arguments it must refuse before a launch and with many shapes to plan.
Either run stops at the first memory or undefined-behaviour error.  Leak
checking is on for the oracle and off for the library, whose CUDA runtime keeps
process-lifetime allocations.
"""
import os
import shutil
import subprocess

import pytest

from gated_delta_rule_64_b200 import build as gdn_build

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
OUT = os.path.join(HERE, "_build", "sanitize")
SAN = ["-fsanitize=address", "-fsanitize=undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer"]


def _stale(target, sources):
    return not os.path.exists(target) or os.path.getmtime(target) < max(os.path.getmtime(s) for s in sources)


def _run(exe, **env):
    e = dict(os.environ, **env)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=600, env=e)
    assert r.returncode == 0, (r.stdout[-3000:], r.stderr[-3000:])
    assert "ERROR: AddressSanitizer" not in r.stderr and "runtime error" not in r.stderr, r.stderr[-3000:]
    return r.stdout


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is needed")
def test_oracle_under_sanitizers():
    os.makedirs(OUT, exist_ok=True)
    exe = os.path.join(OUT, "oracle_san")
    srcs = [os.path.join(ROOT, "oracle", "gdn_oracle.c"), os.path.join(HERE, "csrc", "oracle_sanitize_main.c")]
    if _stale(exe, srcs):
        subprocess.run(["gcc", *SAN, "-g", "-O1", "-pthread", "-fno-fast-math", *srcs, "-o", exe, "-lm"], check=True)
    assert "0 failures" in _run(exe, ASAN_OPTIONS="detect_leaks=1")


def test_library_host_code_under_sanitizers():
    os.makedirs(OUT, exist_ok=True)
    exe = os.path.join(OUT, "abi_san")
    main = os.path.join(HERE, "csrc", "abi_sanitize_main.c")
    if _stale(exe, gdn_build.deps() + [main]):
        objs, procs = [], []
        xc = [a for f in SAN + ["-fPIC"] for a in ("-Xcompiler", f)]
        for src in gdn_build.sources():
            obj = os.path.join(OUT, os.path.basename(src) + ".o")
            objs.append(obj)
            procs.append(subprocess.Popen([gdn_build.nvcc(), *gdn_build.ARCH, "-O1", "-g", "-std=c++17",
                                           "--expt-relaxed-constexpr", *xc, "-I", gdn_build.INCLUDE, "-I",
                                           gdn_build.CSRC, "-c", src, "-o", obj]))
        assert all(p.wait() == 0 for p in procs)
        mobj = os.path.join(OUT, "abi_sanitize_main.o")
        subprocess.run(["gcc", *SAN, "-g", "-I", gdn_build.INCLUDE, "-c", main, "-o", mobj], check=True)
        subprocess.run([gdn_build.nvcc(), *gdn_build.ARCH, *objs, mobj, "-o", exe,
                        *[a for f in SAN for a in ("-Xcompiler", f)]], check=True)
    # (the CUDA driver maps memory where AddressSanitizer keeps its shadow gap)
    assert "0 failures" in _run(exe, ASAN_OPTIONS="detect_leaks=0:protect_shadow_gap=0")
