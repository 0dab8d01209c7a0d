"""Each plausible mistake planted in a copy of the oracle's C source must be
caught by at least one pin.  The copies are built in a temporary directory on
the CPU; the real oracle is untouched."""
import os
import subprocess

import pytest

import oracle
import oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "la_ref.c")

# (name, text in la_ref.c, replacement)
MUTANTS = [
    ("state not decayed", "S[i * Dv + c] = g * S[i * Dv + c] + kt[i] * vt[c];\n        if (j->normalize)",
     "S[i * Dv + c] = S[i * Dv + c] + kt[i] * vt[c];\n        if (j->normalize)"),
    ("decay applied after the add", "S[i * Dv + c] = g * S[i * Dv + c] + kt[i] * vt[c];\n        if (j->normalize)",
     "S[i * Dv + c] = g * (S[i * Dv + c] + kt[i] * vt[c]);\n        if (j->normalize)"),
    ("sign of log decay flipped", "return exp(j->log_g[(size_t)bh * j->T + t]);",
     "return exp(-j->log_g[(size_t)bh * j->T + t]);"),
    ("per-step decay off by one token", "return exp(j->log_g[(size_t)bh * j->T + t]);",
     "return exp(j->log_g[(size_t)bh * j->T + (t > 0 ? t - 1 : 0)]);"),
    ("per-head decay indexed by batch", "return exp(j->log_g[bh % j->H]);",
     "return exp(j->log_g[(bh / j->H) % j->H]);"),
    ("key sum not decayed", "if (j->normalize)\n            for (int i = 0; i < Dk; ++i) z[i] = g * z[i] + kt[i];",
     "if (j->normalize)\n            for (int i = 0; i < Dk; ++i) z[i] = z[i] + kt[i];"),
    ("initial state ignored", "S[a] = j->init_state ? j->init_state[ss + a] : 0.0;", "S[a] = 0.0;"),
    ("initial key sum ignored", "z[a] = (j->normalize && j->init_z) ? j->init_z[sz + a] : 0.0;", "z[a] = 0.0;"),
    ("denominator uses the current key only", "for (int i = 0; i < Dk; ++i) den += qt[i] * z[i];\n        for (int c = 0; c < Dv; ++c) {\n            double num = 0.0;\n            for (int i = 0; i < Dk; ++i) num += qt[i] * S[i * Dv + c];\n            j->out",
     "for (int i = 0; i < Dk; ++i) den += qt[i] * kt[i];\n        for (int c = 0; c < Dv; ++c) {\n            double num = 0.0;\n            for (int i = 0; i < Dk; ++i) num += qt[i] * S[i * Dv + c];\n            j->out"),
    ("state transposed in the read-out", "for (int i = 0; i < Dk; ++i) num += qt[i] * S[i * Dv + c];\n            j->out",
     "for (int i = 0; i < Dk; ++i) num += qt[i] * S[(i * Dv + c) % Dk * Dv + (i * Dv + c) / Dk % Dv];\n            j->out"),
    ("outer product transposed", "S[i * Dv + c] = g * S[i * Dv + c] + kt[i] * vt[c];\n        if (j->normalize)",
     "S[i * Dv + c] = g * S[i * Dv + c] + kt[c % Dk] * vt[i % Dv];\n        if (j->normalize)"),
    ("read-out with the previous token's query", "const double* qt = j->q + sq + (size_t)t * Dk;",
     "const double* qt = j->q + sq + (size_t)(t > 0 ? t - 1 : 0) * Dk;"),
    ("decode state not decayed", "S[i * Dv + c] = g * S[i * Dv + c] + kt[i] * vt[c];\n        if (normalize)",
     "S[i * Dv + c] = S[i * Dv + c] + kt[i] * vt[c];\n        if (normalize)"),
    ("decode per-step decay read per head", "if (decay_kind == 2) g = exp(log_g[bh]);",
     "if (decay_kind == 2) g = exp(log_g[bh % H]);"),
]


def _run_all_pins(lib):
    fwd = lambda *a, **kw: oracle.forward(*a, nthreads=1, lib=lib, **kw)  # noqa: E731
    dec = lambda *a, **kw: oracle.decode_step(*a, lib=lib, **kw)  # noqa: E731
    failed = []
    for check in pins.ALL:
        try:
            check(fwd, dec)
        except AssertionError:
            failed.append(check.__name__)
    try:
        pins.parallel_form(fwd, dec, oracle.parallel_forward)
    except AssertionError:
        failed.append("parallel_form")
    return failed


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {name}"
    path = tmp_path / "la_ref_mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "liblaref_mutant.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o", str(so),
                    str(path), "-lm"], check=True)
    failed = _run_all_pins(oracle.load_library(str(so)))
    assert failed, f"no pin catches the mutant '{name}'"


def test_unmutated_copy_passes(tmp_path):
    so = tmp_path / "liblaref_copy.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o", str(so),
                    SRC, "-lm"], check=True)
    assert _run_all_pins(oracle.load_library(str(so))) == []
