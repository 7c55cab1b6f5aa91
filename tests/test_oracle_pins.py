"""The oracle against its pins (CPU only), and the pins against planted mistakes."""
import functools
import os

import pytest

import oracle
from tests import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "gdn_oracle.c")


def _run_with(lib):
    return functools.partial(oracle.gated_delta_rule, lib=lib, n_threads=2)


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(functools.partial(oracle.gated_delta_rule, n_threads=3))


def test_thread_count_does_not_change_results():
    import numpy as np
    from gated_delta_rule_64_b200.inputs import TINY_F32, make_inputs
    x = make_inputs(TINY_F32.replace(H=5, T=70, h0_std=0.1))
    a = oracle.gated_delta_rule(x.q, x.k, x.v, x.g, x.beta, x.h0, n_threads=1)
    b = oracle.gated_delta_rule(x.q, x.k, x.v, x.g, x.beta, x.h0, n_threads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# Each entry plants one plausible mistake in a copy of the oracle's source.
MUTANTS = {
    "error sign": ("(vt[i] - y[i])", "(vt[i] + y[i])"),
    "no write strength": ("S[i * dk + c] += bt * e * kt[c];", "S[i * dk + c] += e * kt[c];"),
    "gate not exponentiated": ("const double a = exp(J->g[row * H + h]);", "const double a = 1.0 + J->g[row * H + h];"),
    "channel gate on value rows": ("S[i * dk + c] *= al[c];", "S[i * dk + c] *= al[i % dk];"),
    "prediction uses the query": ("acc += S[i * dk + c] * kt[c];", "acc += S[i * dk + c] * qt[c];"),
    "read uses the key": ("acc += S[i * dk + c] * (J->scale * qt[c]);", "acc += S[i * dk + c] * (J->scale * kt[c]);"),
    "snapshot index off by one": ("(t + 1) / J->snapshot_stride - 1;", "(t + 1) / J->snapshot_stride;"),
    "ignores sequence start": ("const int64_t row = start + t;", "const int64_t row = t + 0 * start;"),
    "scale twice": ("acc += S[i * dk + c] * (J->scale * qt[c]);", "acc += S[i * dk + c] * (J->scale * J->scale * qt[c]);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name!r} not found exactly once"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    lib = oracle.bind(oracle.build(force=True, src=str(src), out=str(tmp_path / "mutant.so")))
    run = _run_with(lib)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(run)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name!r}"
