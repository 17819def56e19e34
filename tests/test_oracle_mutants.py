"""The pins must catch plausible mistakes planted in the oracle.

Each mutant is a copy of oracle/kda_oracle.c with one slip pasted in (a dropped term, a wrong sign,
an index on the wrong axis, a wrong constant), compiled with gcc into a temporary library and loaded
through a fresh copy of the oracle's Python binding. Every pin of tests/test_oracle_pins.py is run
against it, and at least one must fail. The unmutated copy, built the same way, must pass them all, so
a failing mutant is the mistake's doing and not the harness's. Mistakes are planted in the oracle, on
the CPU, and never in the product.
"""
import importlib.util
import os
import shutil

import pytest

import test_oracle_pins as pins

HERE = os.path.dirname(os.path.abspath(__file__))
ORACLE_DIR = os.path.join(os.path.dirname(HERE), "oracle")

# (name, text in kda_oracle.c, replacement, number of occurrences replaced)
MUTANTS = [
    ("decay dropped from the state", "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a[i];",
     "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= 1.0;", 1),
    ("decay on the value axis", "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a[i];",
     "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] *= a[j % dk];", 1),
    ("no floor on the log-decay", "exp(fmax((double)lt[i], lfloor))", "exp((double)lt[i])", 1),
    ("floor at 6.7 % instead of 0.67 %", "log(0.0067)", "log(0.067)", 2),
    ("wrong sign of the prediction", "p[j] = bt * ((double)vt[j] - p[j]);", "p[j] = bt * ((double)vt[j] + p[j]);", 1),
    ("beta dropped from the update", "p[j] = bt * ((double)vt[j] - p[j]);", "p[j] = ((double)vt[j] - p[j]);", 1),
    ("prediction read before the decay", "for (int j = 0; j < dv; ++j) p[j] += S[(size_t)i * dv + j] * ki;",
     "for (int j = 0; j < dv; ++j) p[j] += S[(size_t)i * dv + j] * ki / a[i];", 1),
    ("output read with k instead of q", "const double qi = (double)qt[i];", "const double qi = (double)kt[i];", 1),
    ("rank-1 write on the wrong axes", "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += ki * p[j];",
     "for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] += (double)kt[j % dk] * p[i % dv];", 1),
    ("transition without the erase sign", "p[j] = -bt * p[j];", "p[j] = bt * p[j];", 1),
    ("transition without the decay", "for (int j = 0; j < dk; ++j) M[(size_t)i * dk + j] *= a[i];",
     "for (int j = 0; j < dk; ++j) M[(size_t)i * dk + j] *= 1.0;", 1),
    ("compose with M transposed", "acc += Ms[(size_t)i * dk + m] * X[(size_t)m * dv + j];",
     "acc += Ms[(size_t)m * dk + i] * X[(size_t)m * dv + j];", 1),
    ("compose without the zero-start state", "double acc = Zs[(size_t)i * dv + j];", "double acc = 0.0;", 1),
    ("initial state ignored", "    if (s0) memcpy(S, s0, sizeof(double) * (size_t)dk * dv);", "    (void)s0;", 1),
    ("initial state read transposed", "    if (s0) memcpy(S, s0, sizeof(double) * (size_t)dk * dv);",
     "    if (s0) for (int i = 0; i < dk; ++i) for (int j = 0; j < dv; ++j) S[(size_t)i * dv + j] = "
     "s0[(size_t)(j % dk) * dv + (i % dv)];", 1),
    ("E4M3 exponent bias 8", "else mag = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else mag = ldexp(1.0 + (double)m / 8.0, e - 8);", 1),
    ("E4M3 subnormals read as normals", "if (e == 0) mag = ldexp((double)m / 8.0, -6);",
     "if (e == 0) mag = ldexp(1.0 + (double)m / 8.0, -7);", 1),
    ("E4M3 max code read as NaN", "if (e == 15 && m == 7) return NAN;", "if (e == 15 && m >= 6) return NAN;", 1),
    ("E8M0 bias 128", "return ldexp(1.0, (int)e - 127);", "return ldexp(1.0, (int)e - 128);", 1),
    ("shared scale per 16 elements", "scales[r * nb + i / block]", "scales[r * nb + (i / (block / 2)) % nb]", 1),
]


def _pin_calls():
    """Every pin that takes the oracle, with representative parameters for the parametrised ones."""
    calls = []
    for name in dir(pins):
        if not name.startswith("test_"):
            continue
        fn = getattr(pins, name)
        code = fn.__code__
        if "oracle_mod" not in code.co_varnames[:code.co_argcount]:
            continue
        if name == "test_brute_force_dense_products":
            for T, dk, dv in [(7, 5, 3), (16, 8, 6)]:
                calls.append((f"{name}[{T},{dk},{dv}]", lambda m, fn=fn, a=(T, dk, dv): fn(m, *a)))
        elif name == "test_chunk_form_matches_oracle":
            for la in [(-3.0, -0.01), (-5.5, -4.9)]:
                calls.append((f"{name}[64,{la}]", lambda m, fn=fn, la=la: fn(m, 64, la)))
        else:
            calls.append((name, lambda m, fn=fn: fn(m)))
    return calls


def _module_for(src_text, tmp_path, tag):
    d = tmp_path / tag
    d.mkdir()
    src = d / "kda_oracle.c"
    src.write_text(src_text)
    spec = importlib.util.spec_from_file_location(f"oracle_{tag}", os.path.join(ORACLE_DIR, "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(src)
    mod._LIB = str(d / "libkda_oracle.so")
    mod._lib = None
    mod.build(force=True)
    return mod


def _failing_pins(mod):
    failed = []
    for name, call in _pin_calls():
        try:
            call(mod)
        except Exception:   # an assertion, or a bad argument / non-finite value the mistake provoked
            failed.append(name)
    return failed


@pytest.fixture(scope="module")
def original_source():
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not available")
    with open(os.path.join(ORACLE_DIR, "kda_oracle.c")) as f:
        return f.read()


def test_unmutated_copy_passes_every_pin(original_source, tmp_path):
    assert _pin_calls(), "no pins found"
    assert _failing_pins(_module_for(original_source, tmp_path, "clean")) == []


@pytest.mark.parametrize("name,old,new,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_every_planted_mistake_fails_a_pin(original_source, tmp_path, name, old, new, count):
    assert original_source.count(old) >= count, f"mutation site not found: {old}"
    mutated = original_source.replace(old, new, count)
    assert mutated != original_source
    failed = _failing_pins(_module_for(mutated, tmp_path, "mutant"))
    assert failed, f"no pin catches the planted mistake: {name}"
