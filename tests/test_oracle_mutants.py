"""The oracle's pins must be able to fail.

Plausible mistakes are planted, one at a time, in copies of the oracle's
sources: a flipped sign, a wrong index or partner, a dropped term, an operand
taken from the wrong row or segment.  A C mutant is compiled with the oracle's
own gcc flags; a Python mutant (the numpy parts of the oracle) is a copy of
the package module.  A small pytest plugin, loaded only in the subprocesses
this test starts, installs the mutant before the pins import `oracle`: it
sets the oracle's library override (a module attribute) to the compiled C
mutant, or installs the Python mutant as `oracle`.  The CPU
pin suites then run against each mutant in a subprocess.  Every mutant must
make at least one pin fail (pytest exit status 1), while unmodified copies
pass them all, which shows that the harness itself works.  Nothing here
touches a GPU.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_SUITES = ["tests/test_oracle_pins.py", "tests/test_oracle_rope_apply.py"]

# (name, text in rfa_oracle.c, replacement); each text occurs exactly once
MUTANTS = [
    ("rotation_sign", "out[r * D + i] = x1 * c - x2 * s;", "out[r * D + i] = x1 * c + x2 * s;"),
    ("rotation_partner", "x2 = x[r * D + i + half];", "x2 = x[r * D + (i ^ 1) + half];"),
    ("inv_freq_exponent", "pow(base, -2.0 * (double)j / (double)D)", "pow(base, -1.0 * (double)j / (double)D)"),
    ("ntk_exponent", "(double)D / (double)(D - 2)", "(double)D / (double)(D - 1)"),
    ("sincos_column_pairing", "invFreq[(int64_t)b * half + (j % half)]", "invFreq[(int64_t)b * half + (j / 2)]"),
    ("sincos_segment_row", "invFreq[(int64_t)b * half + (j % half)]", "invFreq[(int64_t)(b > 0 ? b - 1 : 0) * half + (j % half)]"),
    ("fp16_exponent_bias", "v = ldexp((double)(1024 + m), e - 25);", "v = ldexp((double)(1024 + m), e - 24);"),
    ("causal_diagonal_dropped", "int32_t jmax = d->causal ? i + 1 : g->len;", "int32_t jmax = d->causal ? i : g->len;"),
    ("softmax_scale_dropped", "s[j] = acc * d->scale;", "s[j] = acc;"),
    ("softmax_not_normalised", "double w = s[j] / z;", "double w = s[j];"),
    ("values_rows_reversed", "const double* vr = g->Vd + (int64_t)j * D;",
     "const double* vr = g->Vd + (int64_t)(jmax - 1 - j) * D;"),
    ("query_not_rotated", "rotate_row(d, xq, p, g->invFreq", "rotate_row(d, xq, 0, g->invFreq"),
    ("gqa_head_map", "rows[3 * r + 1] / G == kvh", "rows[3 * r + 1] % d->Hkv == kvh"),
    ("packed_keys_segment_start", "return ((tok0 + j) * d->Hkv + kh) * (int64_t)d->D;",
     "return ((int64_t)j * d->Hkv + kh) * (int64_t)d->D;"),
    ("adjacent_pair_sign", "out[2 * i] = x1 * c - x2 * s;", "out[2 * i] = x1 * c + x2 * s;"),
    ("rope_op_adjacent_partner", "rx = (j & 1) ? xr[j - 1] : -xr[j + 1];", "rx = (j & 1) ? -xr[j - 1] : xr[j + 1];"),
    ("rope_op_half_partner", "rx = (j < half) ? -xr[j + half] : xr[j - half];",
     "rx = (j < half) ? xr[j + half] : -xr[j - half];"),
    ("rope_op_sin_cos_swapped", "out[r * D + j] = xr[j] * c[j] + rx * s[j];",
     "out[r * D + j] = xr[j] * s[j] + rx * c[j];"),
    ("rms_norm_mean_dropped", "sqrt(ss / (double)D + eps)", "sqrt(ss + eps)"),
    ("rms_norm_gamma_dropped", "out[r * D + j] = gamma[j] * (x[r * D + j] * inv);",
     "out[r * D + j] = (x[r * D + j] * inv);"),
    ("probs_scale_dropped", "p[j] = acc * d->scale;", "p[j] = acc;"),
    ("probs_gqa_head_map", "const int32_t D = d->D, G = d->Hq / d->Hkv, kvh = h / G;",
     "const int32_t D = d->D, G = d->Hq / d->Hkv, kvh = h % d->Hkv;"),
    ("probs_key_at_query_position", "rotate_row(d, x, pk, inv, kr);", "rotate_row(d, x, pq, inv, kr);"),
    ("probs_causal_diagonal_dropped", "int32_t jmax = d->causal ? i + 1 : len;",
     "int32_t jmax = d->causal ? i : len;"),
]


# (name, text in oracle/__init__.py, replacement); each text occurs exactly once
PY_MUTANTS = [
    ("decode_causal_edge", "sc[L - Sq + s + 1:] = -np.inf", "sc[L - Sq + s:] = -np.inf"),
    ("decode_rotation_sign", "z = (x[: D // 2] + 1j * x[D // 2:]) * np.exp(1j * th)",
     "z = (x[: D // 2] + 1j * x[D // 2:]) * np.exp(-1j * th)"),
    ("decode_gqa_map", "kvh = h // G", "kvh = h % Hkv"),
    ("decode_scale_dropped", "sc = (K @ qr) * scale", "sc = (K @ qr)"),
    ("cache_values_from_keys", "vc[sl] = v[t]", "vc[sl] = k[t]"),
    ("cache_norm_skipped", "kn = rms_norm(k.reshape(T * H, D), gamma, eps)", "kn = k.reshape(T * H, D)"),
]

PLUGIN = """import importlib.util, os, sys
if os.environ.get("RFA_MUTANT_PY"):
    _spec = importlib.util.spec_from_file_location("oracle", os.environ["RFA_MUTANT_PY"])
    _mod = importlib.util.module_from_spec(_spec)
    sys.modules["oracle"] = _mod
    _spec.loader.exec_module(_mod)
else:
    import oracle as _mod
_mod._lib_override = os.environ["RFA_MUTANT_LIB"]
"""


def _compile(src: str, path: str) -> None:
    c = path[:-3] + ".c"
    with open(c, "w") as f:
        f.write(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread", c, "-lm", "-o", path])


def _run_pins(lib: str, py=None, plugin_dir=None):
    env = dict(os.environ, RFA_MUTANT_LIB=lib)
    env.pop("RFA_MUTANT_PY", None)
    if py is not None:
        env["RFA_MUTANT_PY"] = py
    env["PYTHONPATH"] = os.pathsep.join([ROOT, plugin_dir] + [p for p in [os.environ.get("PYTHONPATH")] if p])
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-m", "not gpu", "-p", "no:cacheprovider",
                        "-p", "rfa_oracle_mutant_plugin", *PIN_SUITES], cwd=ROOT, env=env, capture_output=True,
                       text=True, timeout=900)
    return r.returncode, (r.stdout + r.stderr)[-1500:]


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    d = str(tmp_path_factory.mktemp("oracle_mutants"))
    with open(oracle._SRC) as f:
        src = f.read()
    with open(os.path.join(os.path.dirname(oracle._SRC), "__init__.py")) as f:
        py_src = f.read()
    with open(os.path.join(d, "rfa_oracle_mutant_plugin.py"), "w") as f:
        f.write(PLUGIN)
    clean = os.path.join(d, "unmodified.so")
    _compile(src, clean)
    jobs = {"unmodified": (clean, None), "unmodified_py": (clean, os.path.join(d, "unmodified_py.py"))}
    with open(jobs["unmodified_py"][1], "w") as f:
        f.write(py_src)
    for name, old, new in MUTANTS:
        assert src.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
        jobs[name] = (os.path.join(d, f"{name}.so"), None)
        _compile(src.replace(old, new), jobs[name][0])
    for name, old, new in PY_MUTANTS:
        assert py_src.count(old) == 1, f"{name}: the text to mutate must occur exactly once"
        jobs[name] = (clean, os.path.join(d, f"{name}.py"))
        with open(jobs[name][1], "w") as f:
            f.write(py_src.replace(old, new))
    names = list(jobs)
    with ThreadPoolExecutor(max_workers=max(1, min(8, os.cpu_count() or 1))) as ex:
        return dict(zip(names, ex.map(lambda n: _run_pins(jobs[n][0], jobs[n][1], d), names)))


@pytest.mark.parametrize("name", ["unmodified", "unmodified_py"])
def test_unmodified_copies_pass_the_pins(results, name):
    rc, out = results[name]
    assert rc == 0, out


@pytest.mark.parametrize("name", [m[0] for m in MUTANTS + PY_MUTANTS])
def test_pins_reject_planted_mistake(results, name):
    rc, out = results[name]
    assert rc == 1, f"{name}: the pins did not fail (exit status {rc})\n{out}"
