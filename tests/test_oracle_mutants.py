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
    ("sign of log decay flipped", "return exp(log_g[(size_t)bh * T + t]);",
     "return exp(-log_g[(size_t)bh * T + t]);"),
    ("per-step decay off by one token", "return exp(log_g[(size_t)bh * T + t]);",
     "return exp(log_g[(size_t)bh * T + (t > 0 ? t - 1 : 0)]);"),
    ("per-head decay indexed by batch", "return exp(log_g[bh % H]);",
     "return exp(log_g[(bh / H) % H]);"),
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
    # backward
    ("state gradient not decayed", "for (int a = 0; a < DD; ++a) G[a] *= g;", "(void)0;"),
    ("key-sum gradient not decayed", "for (int i = 0; i < Dk; ++i) w[i] *= g;", "(void)0;"),
    ("decay gradient against the current state", "for (int a = 0; a < DD; ++a) dg += G[a] * Sp[a];",
     "for (int a = 0; a < DD; ++a) dg += G[a] * St[a];"),
    ("decay gradient without the factor g", "if (j->dlog) j->dlog[(size_t)bh * T + t] = g * dg;",
     "if (j->dlog) j->dlog[(size_t)bh * T + t] = dg;"),
    ("key gradient misses the key-sum term", "j->dk[rq + i] = s + (j->normalize ? w[i] : 0.0);",
     "j->dk[rq + i] = s;"),
    ("denominator gradient sign flipped", "f = -dn / (den * den);", "f = dn / (den * den);"),
    ("value gradient from the query", "for (int i = 0; i < Dk; ++i) s += G[i * Dv + c] * kt[i];",
     "for (int i = 0; i < Dk; ++i) s += G[i * Dv + c] * qt[i];"),
    ("query gradient from the previous state", "for (int c = 0; c < Dv; ++c) s += St[i * Dv + c] * e[c];",
     "for (int c = 0; c < Dv; ++c) s += Sp[i * Dv + c] * e[c];"),
    ("final state gradient ignored", "G[a] = j->d_final_state ? j->d_final_state[ss + a] : 0.0;", "G[a] = 0.0;"),
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
    bwd = lambda *a, **kw: oracle.backward(*a, nthreads=1, lib=lib, **kw)  # noqa: E731
    real_fwd = lambda *a, **kw: oracle.forward(*a, nthreads=1, **kw)  # noqa: E731
    for name, run in (("backward_finite_differences", lambda: pins.backward_finite_differences(bwd, real_fwd)),
                      ("backward_t1_closed_form", lambda: pins.backward_t1_closed_form(bwd)),
                      ("backward_parallel_form", lambda: pins.backward_parallel_form(bwd, real_fwd))):
        try:
            run()
        except AssertionError:
            failed.append(name)
    return failed


WKV4_SRC = os.path.join(os.path.dirname(oracle.__file__), "wkv4_ref.c")

# (name, text in wkv4_ref.c, replacement)
WKV4_MUTANTS = [
    ("bonus left out of the read-out", "out[i] = mean + sigmoid(u[c] + kt - logw) * (vt - mean);",
     "out[i] = mean + sigmoid(kt - logw) * (vt - mean);"),
    ("state not decayed", "const double decayed = logw + w[c];", "const double decayed = logw;"),
    ("bonus used in the update", "mean += sigmoid(kt - decayed) * (vt - mean);",
     "mean += sigmoid(u[c] + kt - decayed) * (vt - mean);"),
    ("read-out ignores the state", "out[i] = mean + sigmoid(u[c] + kt - logw) * (vt - mean);", "out[i] = vt;"),
    ("total weight not carried", "logw = logaddexp(decayed, kt);", "logw = kt;"),
    ("empty state at weight 1", "double mean = 0.0, logw = -INFINITY;", "double mean = 0.0, logw = 0.0;"),
    ("logistic of the wrong sign", "if (x >= 0.0) return 1.0 / (1.0 + exp(-x));", "if (x >= 0.0) return 1.0 / (1.0 + exp(x));"),
    ("sum of weights as their maximum", "return hi + log1p(exp(lo - hi));", "return hi;"),
    ("carried state's scale ignored", "logw = init_state[s + 2 * C] + log(init_state[s + C]);",
     "logw = log(init_state[s + C]);"),
    ("final mean written as the sum", "final_state[s] = empty ? 0.0 : mean;", "final_state[s] = empty ? 0.0 : mean * exp(logw);"),
]


def _run_wkv4_pins(lib):
    wkv = lambda *a: oracle.wkv4(*a, lib=lib)  # noqa: E731
    failed = []
    for check in pins.WKV4:
        try:
            check(wkv, oracle.wkv4_direct)
        except AssertionError:
            failed.append(check.__name__)
    return failed


EMA_SRC = os.path.join(os.path.dirname(oracle.__file__), "ema_ref.c")

# (name, text in ema_ref.c, replacement)
EMA_MUTANTS = [
    ("factor ignored", "s = f[i] * s + x[i];", "s = s + x[i];"),
    ("decay after the add", "s = f[i] * s + x[i];", "s = f[i] * (s + x[i]);"),
    ("factor of the previous step", "s = f[i] * s + x[i];",
     "s = f[i > (size_t)C ? i - C : i] * s + x[i];"),
    ("reverse runs forward", "const int t = reverse ? T - 1 - step : step;", "const int t = step;"),
    ("carried state ignored", "double s = init_state ? init_state[(size_t)b * C + c] : 0.0;", "double s = 0.0;"),
]


def _run_ema_pins(lib):
    fn = lambda *a, **kw: oracle.ema(*a, lib=lib, **kw)  # noqa: E731
    failed = []
    for check in pins.EMA:
        try:
            check(fn)
        except AssertionError:
            failed.append(check.__name__)
    return failed


@pytest.mark.parametrize("name,old,new", EMA_MUTANTS, ids=[m[0] for m in EMA_MUTANTS])
def test_ema_mutant_is_caught(tmp_path, name, old, new):
    src = open(EMA_SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {name}"
    failed = _run_ema_pins(_build_copy(tmp_path, ema_text=src.replace(old, new)))
    assert failed, f"no pin catches the mutant '{name}'"


def test_ema_unmutated_copy_passes(tmp_path):
    assert _run_ema_pins(_build_copy(tmp_path)) == []


def _build_copy(tmp_path, wkv4_text=None, ema_text=None):
    paths = []
    for src in (SRC, WKV4_SRC, EMA_SRC):
        p = tmp_path / os.path.basename(src)
        text = open(src).read()
        if src == WKV4_SRC and wkv4_text is not None:
            text = wkv4_text
        if src == EMA_SRC and ema_text is not None:
            text = ema_text
        p.write_text(text)
        paths.append(str(p))
    so = tmp_path / "liblaref_copy.so"
    subprocess.run(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread", "-o", str(so), *paths, "-lm"],
                   check=True)
    return oracle.load_library(str(so))


@pytest.mark.parametrize("name,old,new", WKV4_MUTANTS, ids=[m[0] for m in WKV4_MUTANTS])
def test_wkv4_mutant_is_caught(tmp_path, name, old, new):
    src = open(WKV4_SRC).read()
    assert src.count(old) == 1, f"mutation site not unique: {name}"
    failed = _run_wkv4_pins(_build_copy(tmp_path, src.replace(old, new)))
    assert failed, f"no pin catches the mutant '{name}'"


def test_wkv4_unmutated_copy_passes(tmp_path):
    assert _run_wkv4_pins(_build_copy(tmp_path)) == []


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
