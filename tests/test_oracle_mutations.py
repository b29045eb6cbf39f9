"""Plant plausible mistakes in copies of the oracle (CPU only) and check that
the pins catch every one: a dropped term, a wrong operand, a missing factor."""
import inspect
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "la_oracle.c")

MUTANTS = {
    "undecayed_normaliser": ("z[i] = gamma * z[i] + b[i];", "z[i] = z[i] + b[i];"),
    "query_written_to_state": ("Si[j] = gamma * Si[j] + b[i] * vt[j];", "Si[j] = gamma * Si[j] + a[i] * vt[j];"),
    "key_reads_state": ("num += a[i] * S[(size_t)i * dv + j];", "num += b[i] * S[(size_t)i * dv + j];"),
    "no_eps": ("den += eps;", ""),
    "elu_without_plus_one": ("x > 0.0 ? x + 1.0 : exp(x)", "x > 0.0 ? x : exp(x)"),
    "error_on_undecayed_state": ("(vt[j] - at * vhat[j])", "(vt[j] - vhat[j])"),
    "delta_without_decay": ("Si[j] = at * Si[j] + gt", "Si[j] = Si[j] + gt"),
    "delta_reads_with_key": ("for (int i = 0; i < d; ++i) s += S[(size_t)i * dv + j] * qt[i];",
                             "for (int i = 0; i < d; ++i) s += S[(size_t)i * dv + j] * kt[i];"),
    "delta_gate_dropped": ("gt * kt[i] * (vt[j]", "kt[i] * (vt[j]"),
    "gla_gate_on_value_dim": ("Si[j] = at[i] * Si[j] + kt[i] * vt[j];", "Si[j] = at[j % d] * Si[j] + kt[i] * vt[j];"),
    "gla_gate_after_write": ("Si[j] = at[i] * Si[j] + kt[i] * vt[j];", "Si[j] = at[i] * (Si[j] + kt[i] * vt[j]);"),
    "gla_reads_with_key": ("for (int i = 0; i < d; ++i) acc += qt[i] * S[(size_t)i * dv + j];",
                           "for (int i = 0; i < d; ++i) acc += kt[i] * S[(size_t)i * dv + j];"),
    "conv_reversed_taps": ("W[((size_t)h * d + c) * w + i] * XH(t + i, c)",
                           "W[((size_t)h * d + c) * w + (w - 1 - i)] * XH(t + i, c)"),
    "conv_window_off_by_one": ("acc += W[((size_t)h * d + c) * w + i] * XH(t + i, c);",
                               "acc += W[((size_t)h * d + c) * w + i] * XH(t + i + 1 < N + hist ? t + i + 1 : t + i, c);"),
    "conv_cache_ignored": ("(cc ? cc[(size_t)(r) * d + (c)] : 0.0)", "0.0"),
}


def _pin_tests():
    out = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        marks = getattr(fn, "pytestmark", [])
        params = [m for m in marks if m.name == "parametrize"]
        if params:
            argnames, values = params[0].args[0], params[0].args[1]
            names = [a.strip() for a in argnames.split(",")]
            for val in values:
                val = val if isinstance(val, tuple) else (val,)
                out.append((name, fn, dict(zip(names, val))))
        else:
            out.append((name, fn, {}))
    return out


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_mutant(mutant, tmp_path):
    old, new = MUTANTS[mutant]
    src = open(SRC).read()
    assert src.count(old) == 1, mutant
    mpath = tmp_path / "la_oracle.c"
    mpath.write_text(src.replace(old, new))
    (tmp_path / "la_oracle.h").write_text(open(SRC[:-2] + ".h").read())
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-ffp-contract=off",
                    str(mpath), "-o", str(lib), "-lm"], check=True)
    caught = []
    oracle._use_library(str(lib))
    try:
        for name, fn, kwargs in _pin_tests():
            if "golden" in inspect.signature(fn).parameters:
                from tests.conftest import read_golden
                kwargs = dict(kwargs, golden=read_golden)
            try:
                fn(**kwargs)
            except AssertionError:
                caught.append(name)
    finally:
        oracle._use_library(None)
    assert caught, f"no pin catches mutant {mutant}"
