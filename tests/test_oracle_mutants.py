"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), compiles it, points the oracle module at that
library and runs every oracle pin (the parametrised test functions of the
pin files, called directly): at least one pin must fail.  The unchanged
source, compiled the same way, must pass them all, so a failure under a
mistake comes from the mistake and not from the harness.

The mistakes follow the steps of the method in the paper note "Reformer"
(eightmm.github.io): the hash ("LSH Attention", hash equation), the stable
sort and the chunk window ("Sorting and Chunking"), unit keys and the score
scale ("Shared Query-Key Space"; output equation), the self and causal
masks ("Implementation Reading"), the round merge ("Multiple Hash Rounds"),
the backward, and the optional readings.
"""
import importlib.util
import inspect
import itertools
import os
import subprocess

import pytest

from oracle import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "lsh_oracle.c")
PIN_FILES = ("test_oracle_pins.py", "test_oracle_pins_props.py", "test_oracle_pins_flags.py",
             "test_oracle_pins_local.py", "test_oracle_pins_rev.py")

# (name, text in the source, its replacement, which occurrence (0-based) or None for the only one)
MUTANTS = [
    ("hash: halves of [xR ; -xR] exchanged",
     "u[k] = p;\n            u[half + k] = -p;", "u[k] = -p;\n            u[half + k] = p;", None),
    ("hash: last maximum kept on a tie",
     "if (u[k] > u[best]) best = k;", "if (u[k] >= u[best]) best = k;", None),
    ("hash: rotation read transposed",
     "p += xi[t] * Rr[(size_t)t * half + k];", "p += xi[t] * Rr[(size_t)k * d + t];", None),
    ("sort: buckets in descending order",
     "return (x > y) - (x < y);", "return (x < y) - (x > y);", None),
    ("keys: not unit-normalised",
     "nj > 0.0 ? x[(size_t)j * d + t] / nj : 0.0;", "x[(size_t)j * d + t];", None),
    ("forward: no 1/sqrt(d) scale",
     "const double tau = 1.0 / sqrt((double)d);", "const double tau = 1.0;", 0),
    ("backward: no 1/sqrt(d) scale",
     "const double tau = 1.0 / sqrt((double)d);", "const double tau = 1.0;", 1),
    ("window: previous chunk left out",
     "long w0 = (c - before) * m;", "long w0 = (c - before + 1) * m;", None),
    ("window: own chunk left out",
     "long w1 = (c + after + 1) * m;", "long w1 = (c + after) * m;", None),
    ("window: shifted one chunk on (c and c+1)",
     "long w0 = (c - before) * m;\n    if (w0 < 0) w0 = 0;\n    long w1 = (c + after + 1) * m;",
     "long w0 = (c - before + 1) * m;\n    if (w0 < 0) w0 = 0;\n    long w1 = (c + after + 2) * m;", None),
    ("causal: masked on sorted slots",
     "if (causal && j > i) continue;", "if (causal && t > s) continue;", None),
    ("self: never removed",
     "if (t == s) continue;", "if (t == s && 0) continue;", None),
    ("self: not kept when nothing else is left",
     "if (self_penalty || nc == 0) {", "if (self_penalty) {", None),
    ("merge: uniform average of the rounds",
     "double w = exp(lse[(size_t)r * L + i] - big);", "double w = 1.0 / R;", None),
    ("merge: weights not normalised",
     "double big = mx + log(s);", "double big = mx;", None),
    ("backward: sign of delta",
     "double dz = p * (gv - delta);", "double dz = p * (gv + delta);", None),
    ("backward: per-round weights instead of the merged softmax",
     "double p = exp(tau * dot - big[i]);", "double p = exp(tau * dot - lse[(size_t)r * L + i]);", None),
    ("backward: key role not projected off the key direction",
     "dx[(size_t)j * d + t] += (gj[t] - kj[t] * kg) / norm[j];", "dx[(size_t)j * d + t] += gj[t] / norm[j];",
     None),
    ("backward: key role left out",
     "dk[(size_t)j * d + t] += dz * tau * xi[t];", "dk[(size_t)j * d + t] += 0.0 * xi[t];", None),
    ("bucket mask: buckets compared by slot",
     "if (bucket && bucket[j] != bucket[i]) continue;", "if (bucket && bucket[t] != bucket[s]) continue;", None),
    ("self penalty: score of the wrong sign",
     "#define ORACLE_SELF_PENALTY (-1.0e5)", "#define ORACLE_SELF_PENALTY (1.0e5)", None),
]


def _load_pins():
    """Every (function, arguments) of the pin files, parametrisations expanded."""
    pins = []
    for fname in PIN_FILES:
        spec = importlib.util.spec_from_file_location("_pins_" + fname[:-3], os.path.join(HERE, fname))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        for name, fn in vars(mod).items():
            if not (name.startswith("test_") and inspect.isfunction(fn)):
                continue
            axes = []
            for mark in getattr(fn, "pytestmark", []):
                if mark.name != "parametrize":
                    continue
                names = mark.args[0]
                names = [n.strip() for n in names.split(",")] if isinstance(names, str) else list(names)
                rows = []
                for val in mark.args[1]:
                    val = getattr(val, "values", val)              # pytest.param
                    rows.append(dict(zip(names, (val,) if len(names) == 1 else val)))
                axes.append(rows)
            for combo in itertools.product(*axes):
                kwargs = {}
                for part in combo:
                    kwargs.update(part)
                assert set(kwargs) == set(inspect.signature(fn).parameters), (fname, name)
                pins.append((f"{fname}::{name}{sorted(kwargs.items())}", fn, kwargs))
    return pins


def _build(text, path):
    csrc = path + ".c"
    with open(csrc, "w") as f:
        f.write(text)
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-shared", "-fPIC", "-o", path, csrc, "-lm"])
    return path


def _failing_pin(lib_path, pins):
    """Runs the pins against the library at lib_path; returns the first pin
    that fails (its name), or None when all pass."""
    saved = oracle._lib
    oracle._lib = oracle.open_library(lib_path)
    try:
        for name, fn, kwargs in pins:
            try:
                fn(**kwargs)
            except Exception:          # an assertion, or an error a wrong value leads to
                return name
        return None
    finally:
        oracle._lib = saved


@pytest.fixture(scope="module")
def pins():
    return _load_pins()


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


def test_unchanged_source_passes_every_pin(pins, source, tmp_path_factory):
    assert len(pins) > 80
    path = _build(source, str(tmp_path_factory.mktemp("oracle_copy") / "liboracle_copy.so"))
    assert _failing_pin(path, pins) is None


@pytest.mark.parametrize("name,old,new,which", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_fails_a_pin(pins, source, tmp_path_factory, name, old, new, which):
    n = source.count(old)
    if which is None:
        assert n == 1, (name, n)
        text = source.replace(old, new)
    else:
        assert n > which, (name, n)
        at = -1
        for _ in range(which + 1):
            at = source.index(old, at + 1)
        text = source[:at] + new + source[at + len(old):]
    path = _build(text, str(tmp_path_factory.mktemp("oracle_mutant") / "liboracle_mutant.so"))
    assert _failing_pin(path, pins) is not None, f"no pin fails with the mistake: {name}"
